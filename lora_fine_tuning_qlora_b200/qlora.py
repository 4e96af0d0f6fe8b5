"""Python binding of libqlora.so: the C ABI of include/qlora.h, same names.

Argument marshalling only: every function checks dtypes/shapes of the torch
tensors it is given, passes their device pointers and the current CUDA stream
to the library, and raises ``QLoraError`` on a non-OK status.  All arithmetic
runs in the library's kernels; there is no fallback of any kind.  If the
library has not been built, importing this module raises.

PyTorch only provides device memory and streams here.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_F32 = 0
QLORA_BF16 = 1

STATUS = {0: "QLORA_OK", -1: "QLORA_EINVAL", -2: "QLORA_EALIGN", -3: "QLORA_ESHAPE",
          -4: "QLORA_ECUDA", -5: "QLORA_EUNSUPPORTED", -6: "QLORA_ETIMEOUT"}

EXPORTED = ("qlora_quantize_weight", "qlora_workspace_bytes", "qlora_forward",
            "qlora_backward", "qlora_merge", "qlora_last_error", "qlora_device_status",
            "qlora_version", "qlora_relu", "qlora_relu_backward", "qlora_quantize_input",
            "qlora_gemm_forward", "qlora_lora_grad_dy", "qlora_gemm_dx", "qlora_lora_grad_x",
            "qlora_selftest_wait_timeout", "qlora_backward_noalloc", "qlora_lora_g",
            "qlora_lora_grad_b", "qlora_gemm_forward_relu", "qlora_gemm_dx_relu",
            "qlora_set_rank_pass_rows", "qlora_quantize_weight_int4", "qlora_unpack_int4",
            "qlora_gemm_dx_int4", "qlora_merge_int4", "qlora_gemm_forward_int4",
            "qlora_outlier_cap", "qlora_outlier_workspace_bytes", "qlora_outlier_quantize",
            "qlora_outlier_forward", "qlora_outlier_backward", "qlora_permute",
            "qlora_fp8_quantize", "qlora_fp8_gemm", "qlora_fp8_colsum_workspace_bytes",
            "qlora_fp8_quantize_colsum", "qlora_fp8_gemm_workspace_bytes", "qlora_fp8_gemm_ws")


class QLoraError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s (%d): %s" % (STATUS.get(code, "?"), code, msg))
        self.code = code


class LayerDesc(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("N", ctypes.c_int), ("r", ctypes.c_int),
                ("alpha", ctypes.c_float), ("act_dtype", ctypes.c_int)]


class Debug(ctypes.Structure):
    _fields_ = [("xq", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("acc", ctypes.c_void_p)]


class OutlierKernelStruct(ctypes.Structure):
    """qlora_outlier_kernel: device pointers of an outlier-compensated kernel."""
    _fields_ = [("codes_nk", ctypes.c_void_p), ("codes_kn", ctypes.c_void_p),
                ("par", ctypes.c_void_p), ("start_nk", ctypes.c_void_p),
                ("ent_nk", ctypes.c_void_p), ("start_kn", ctypes.c_void_p),
                ("ent_kn", ctypes.c_void_p), ("cap", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libqlora.so is not built (run python -m lora_fine_tuning_qlora_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.qlora_quantize_weight.argtypes = [P, I, I, P, P, P]
    lib.qlora_quantize_weight.restype = I
    lib.qlora_workspace_bytes.argtypes = [ctypes.POINTER(LayerDesc), I]
    lib.qlora_workspace_bytes.restype = ctypes.c_size_t
    lib.qlora_forward.argtypes = [ctypes.POINTER(LayerDesc), I, P, P, P, P, P, P, P, P, P,
                                  ctypes.c_size_t, ctypes.POINTER(Debug), P]
    lib.qlora_forward.restype = I
    lib.qlora_backward.argtypes = [ctypes.POINTER(LayerDesc), I, P, P, P, P, P, P, P, P, P, P,
                                   P, P, ctypes.c_size_t, P]
    lib.qlora_backward.restype = I
    lib.qlora_backward_noalloc.argtypes = [ctypes.POINTER(LayerDesc), I, P, P, P, P, P, P, P, P,
                                           P, P, P, P]
    lib.qlora_backward_noalloc.restype = I
    lib.qlora_merge.argtypes = [ctypes.POINTER(LayerDesc), P, P, P, P, P, P, P]
    lib.qlora_merge.restype = I
    lib.qlora_last_error.restype = ctypes.c_char_p
    lib.qlora_device_status.argtypes = [P]
    lib.qlora_device_status.restype = I
    lib.qlora_version.restype = ctypes.c_char_p
    lib.qlora_relu.argtypes = [P, ctypes.c_size_t, I, P]
    lib.qlora_relu.restype = I
    lib.qlora_relu_backward.argtypes = [P, P, ctypes.c_size_t, I, P]
    lib.qlora_relu_backward.restype = I
    D = ctypes.POINTER(LayerDesc)
    Z = ctypes.c_size_t
    lib.qlora_quantize_input.argtypes = [D, I, P, P, P, P, P, P]
    lib.qlora_gemm_forward.argtypes = [D, I, P, P, P, P, P, P, P, P, P, P]
    lib.qlora_lora_grad_dy.argtypes = [D, I, P, P, P, P, P, P, P, Z, P]
    lib.qlora_lora_g.argtypes = [D, I, P, P, P, Z, P]
    lib.qlora_lora_grad_b.argtypes = [D, I, P, P, P, P, P]
    lib.qlora_gemm_dx.argtypes = [D, I, P, P, P, P, P, P, Z, P]
    lib.qlora_gemm_forward_relu.argtypes = [D, I, P, P, P, P, P, P, P, P, P, P]
    lib.qlora_gemm_dx_relu.argtypes = [D, I, P, P, P, P, P, P, P, Z, P]
    lib.qlora_lora_grad_x.argtypes = [D, I, P, P, P, Z, P]
    for f in (lib.qlora_quantize_input, lib.qlora_gemm_forward, lib.qlora_lora_grad_dy,
              lib.qlora_lora_g, lib.qlora_lora_grad_b, lib.qlora_gemm_dx, lib.qlora_lora_grad_x,
              lib.qlora_gemm_forward_relu, lib.qlora_gemm_dx_relu):
        f.restype = I
    lib.qlora_quantize_weight_int4.argtypes = [P, I, I, P, P, P]
    lib.qlora_unpack_int4.argtypes = [P, I, I, P, P]
    lib.qlora_gemm_dx_int4.argtypes = [D, I, P, P, P, P, P, P, Z, P]
    lib.qlora_gemm_forward_int4.argtypes = [D, I, P, P, P, P, P, P, P, P, P, P]
    lib.qlora_gemm_forward_int4.restype = I
    lib.qlora_merge_int4.argtypes = [D, P, P, P, P, P, P, P]
    for f in (lib.qlora_quantize_weight_int4, lib.qlora_unpack_int4, lib.qlora_gemm_dx_int4,
              lib.qlora_merge_int4):
        f.restype = I
    OK = ctypes.POINTER(OutlierKernelStruct)
    lib.qlora_outlier_cap.argtypes = [I, I]
    lib.qlora_outlier_cap.restype = Z
    lib.qlora_outlier_workspace_bytes.argtypes = [I, I]
    lib.qlora_outlier_workspace_bytes.restype = Z
    lib.qlora_outlier_quantize.argtypes = [P, I, I, OK, P, Z, P]
    lib.qlora_outlier_forward.argtypes = [D, I, P, OK, P, P, P, P, P, P, Z, P]
    lib.qlora_outlier_backward.argtypes = [D, I, P, P, OK, P, P, P, P, P, P, P, P, Z, P]
    for f in (lib.qlora_outlier_quantize, lib.qlora_outlier_forward, lib.qlora_outlier_backward):
        f.restype = I
    lib.qlora_fp8_quantize.argtypes = [P, I, I, I, I, P, P, P, I, P, P, P, Z, P]
    lib.qlora_fp8_quantize.restype = I
    lib.qlora_fp8_colsum_workspace_bytes.argtypes = [I, I]
    lib.qlora_fp8_colsum_workspace_bytes.restype = Z
    lib.qlora_fp8_quantize_colsum.argtypes = [P, I, I, I, I, P, P, P, I, P, P, P, P, Z, P]
    lib.qlora_fp8_quantize_colsum.restype = I
    lib.qlora_fp8_gemm.argtypes = [P, I, P, I, I, I, I, P, P, P, P, I, P]
    lib.qlora_fp8_gemm_workspace_bytes.argtypes = [I, I, I]
    lib.qlora_fp8_gemm_workspace_bytes.restype = Z
    lib.qlora_fp8_gemm_ws.argtypes = [P, I, P, I, I, I, I, P, P, P, P, I, P, Z, P]
    lib.qlora_fp8_gemm_ws.restype = I
    lib.qlora_fp8_gemm.restype = I
    lib.qlora_permute.argtypes = [P, P, I, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int), I, P]
    lib.qlora_permute.restype = I
    lib.qlora_set_rank_pass_rows.argtypes = [I]
    lib.qlora_set_rank_pass_rows.restype = I
    lib.qlora_selftest_wait_timeout.argtypes = [ctypes.c_uint, P]
    lib.qlora_selftest_wait_timeout.restype = I
    return lib


_lib = _load()


def lib():
    return _lib


def _check(code: int):
    if code != 0:
        raise QLoraError(code, _lib.qlora_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def act_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return QLORA_BF16
    if dtype == torch.float32:
        return QLORA_F32
    raise ValueError("activations must be float32 or bfloat16")


def desc(K: int, N: int, r: int, alpha: float, act: torch.dtype) -> LayerDesc:
    return LayerDesc(int(K), int(N), int(r), float(alpha), act_code(act))


def version() -> str:
    return _lib.qlora_version().decode()


def qlora_workspace_bytes(d: LayerDesc, M: int) -> int:
    return int(_lib.qlora_workspace_bytes(ctypes.byref(d), int(M)))


def workspace(d: LayerDesc, M: int, device=None) -> torch.Tensor:
    """A uint8 device buffer big enough for forward and backward at M tokens."""
    n = qlora_workspace_bytes(d, M)
    if n == 0:
        raise QLoraError(-1, "invalid layer descriptor")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def qlora_quantize_weight(W: torch.Tensor, Wq: torch.Tensor, sw: torch.Tensor, stream=None):
    K, N = W.shape
    assert W.dtype == torch.float32 and Wq.dtype == torch.int8 and sw.dtype == torch.float32
    assert tuple(Wq.shape) == (N, K) and tuple(sw.shape) == (N,)
    _check(_lib.qlora_quantize_weight(_ptr(W), K, N, _ptr(Wq), _ptr(sw), _stream(stream)))


def quantize_weight(W: torch.Tensor, stream=None):
    K, N = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    sw = torch.empty((N,), dtype=torch.float32, device=W.device)
    qlora_quantize_weight(W, Wq, sw, stream)
    return Wq, sw


def qlora_forward(d: LayerDesc, M: int, X, Wq, sw, bias, A, B, Y, xA, ws, dbg: Optional[Debug] = None,
                  stream=None):
    _check(_lib.qlora_forward(ctypes.byref(d), int(M), _ptr(X), _ptr(Wq), _ptr(sw), _ptr(bias),
                              _ptr(A), _ptr(B), _ptr(Y), _ptr(xA), _ptr(ws), ws.numel(),
                              ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))


def qlora_backward(d: LayerDesc, M: int, X, dY, Wq, sw, A, B, xA, dX, dA, dB, dbias, ws,
                   stream=None):
    _check(_lib.qlora_backward(ctypes.byref(d), int(M), _ptr(X), _ptr(dY), _ptr(Wq), _ptr(sw),
                               _ptr(A), _ptr(B), _ptr(xA), _ptr(dX), _ptr(dA), _ptr(dB),
                               _ptr(dbias), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_backward_noalloc(d: LayerDesc, M: int, X, dY, Wq, sw, A, B, xA, dX, dA, dB, dbias,
                           stream=None):
    """qlora_backward with the library's static scratch instead of a workspace."""
    _check(_lib.qlora_backward_noalloc(ctypes.byref(d), int(M), _ptr(X), _ptr(dY), _ptr(Wq),
                                       _ptr(sw), _ptr(A), _ptr(B), _ptr(xA), _ptr(dX), _ptr(dA),
                                       _ptr(dB), _ptr(dbias), _stream(stream)))


def qlora_merge(d: LayerDesc, Wq, sw, A, B, Wq_out, sw_out, stream=None):
    _check(_lib.qlora_merge(ctypes.byref(d), _ptr(Wq), _ptr(sw), _ptr(A), _ptr(B), _ptr(Wq_out),
                            _ptr(sw_out), _stream(stream)))


def qlora_quantize_input(d: LayerDesc, M: int, X, A, Xq, sx, xA, stream=None):
    _check(_lib.qlora_quantize_input(ctypes.byref(d), int(M), _ptr(X), _ptr(A), _ptr(Xq), _ptr(sx),
                                     _ptr(xA), _stream(stream)))


def qlora_gemm_forward(d: LayerDesc, M: int, Xq, sx, Wq, sw, bias, xA, B, Y, acc=None, stream=None):
    _check(_lib.qlora_gemm_forward(ctypes.byref(d), int(M), _ptr(Xq), _ptr(sx), _ptr(Wq), _ptr(sw),
                                   _ptr(bias), _ptr(xA), _ptr(B), _ptr(Y), _ptr(acc), _stream(stream)))


def qlora_lora_grad_dy(d: LayerDesc, M: int, dY, B, xA, dB, dbias, ws, G=None, stream=None):
    """dB, dbias; leaves G in `ws` for qlora_gemm_dx / qlora_lora_grad_x (and
    writes the summed G too when a tensor is given)."""
    _check(_lib.qlora_lora_grad_dy(ctypes.byref(d), int(M), _ptr(dY), _ptr(B), _ptr(xA), _ptr(dB),
                                   _ptr(dbias), _ptr(G), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_gemm_forward_relu(d: LayerDesc, M: int, Xq, sx, Wq, sw, bias, xA, B, Y, acc=None,
                            stream=None):
    """qlora_gemm_forward with the following ReLU in its epilogue."""
    _check(_lib.qlora_gemm_forward_relu(ctypes.byref(d), int(M), _ptr(Xq), _ptr(sx), _ptr(Wq),
                                        _ptr(sw), _ptr(bias), _ptr(xA), _ptr(B), _ptr(Y), _ptr(acc),
                                        _stream(stream)))


def qlora_gemm_dx_relu(d: LayerDesc, M: int, dY, Wq, sw, A, X, dX, ws, stream=None):
    """qlora_gemm_dx taken back through the ReLU that produced X."""
    _check(_lib.qlora_gemm_dx_relu(ctypes.byref(d), int(M), _ptr(dY), _ptr(Wq), _ptr(sw), _ptr(A),
                                   _ptr(X), _ptr(dX), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_lora_g(d: LayerDesc, M: int, dY, B, ws, stream=None):
    """G = dY B^T into `ws` (the first half of qlora_lora_grad_dy)."""
    _check(_lib.qlora_lora_g(ctypes.byref(d), int(M), _ptr(dY), _ptr(B), _ptr(ws), ws.numel(),
                             _stream(stream)))


def qlora_lora_grad_b(d: LayerDesc, M: int, dY, xA, dB, dbias, stream=None):
    """dB and dbias (the second half of qlora_lora_grad_dy)."""
    _check(_lib.qlora_lora_grad_b(ctypes.byref(d), int(M), _ptr(dY), _ptr(xA), _ptr(dB),
                                  _ptr(dbias), _stream(stream)))


def qlora_gemm_dx(d: LayerDesc, M: int, dY, Wq, sw, A, dX, ws, stream=None):
    _check(_lib.qlora_gemm_dx(ctypes.byref(d), int(M), _ptr(dY), _ptr(Wq), _ptr(sw), _ptr(A),
                              _ptr(dX), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_lora_grad_x(d: LayerDesc, M: int, X, dA, ws, stream=None):
    _check(_lib.qlora_lora_grad_x(ctypes.byref(d), int(M), _ptr(X), _ptr(dA), _ptr(ws), ws.numel(),
                                  _stream(stream)))


def quantize_weight_int4(W: torch.Tensor, stream=None):
    """W [K, N] fp32 -> (Wp [N, K/2] uint8 packed int4 codes, sw [N] fp32)."""
    K, N = W.shape
    W = W.float().contiguous()
    Wp = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    sw = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check(_lib.qlora_quantize_weight_int4(_ptr(W), K, N, _ptr(Wp), _ptr(sw), _stream(stream)))
    return Wp, sw


def unpack_int4(Wp: torch.Tensor, stream=None) -> torch.Tensor:
    """Wp [N, K/2] -> int8 codes [N, K] (the forward's Wq)."""
    N, K2 = Wp.shape
    Wq = torch.empty((N, 2 * K2), dtype=torch.int8, device=Wp.device)
    _check(_lib.qlora_unpack_int4(_ptr(Wp), 2 * K2, N, _ptr(Wq), _stream(stream)))
    return Wq


def qlora_gemm_forward_int4(d: LayerDesc, M: int, Xq, sx, Wp, sw, bias, xA, B, Y, acc=None,
                            stream=None):
    """qlora_gemm_forward on packed int4 codes Wp [N, K/2]."""
    _check(_lib.qlora_gemm_forward_int4(ctypes.byref(d), int(M), _ptr(Xq), _ptr(sx), _ptr(Wp),
                                        _ptr(sw), _ptr(bias), _ptr(xA), _ptr(B), _ptr(Y), _ptr(acc),
                                        _stream(stream)))


def qlora_gemm_dx_int4(d: LayerDesc, M: int, dY, Wp, sw, A, dX, ws, stream=None):
    _check(_lib.qlora_gemm_dx_int4(ctypes.byref(d), int(M), _ptr(dY), _ptr(Wp), _ptr(sw), _ptr(A),
                                   _ptr(dX), _ptr(ws), ws.numel(), _stream(stream)))


def merge_int4(d: LayerDesc, Wp, sw, A, B, stream=None):
    """Lossy merge of an int4 layer -> (Wp' [N, K/2], sw' [N])."""
    Wp2 = torch.empty_like(Wp)
    sw2 = torch.empty_like(sw)
    _check(_lib.qlora_merge_int4(ctypes.byref(d), _ptr(Wp), _ptr(sw), _ptr(A), _ptr(B), _ptr(Wp2),
                                 _ptr(sw2), _stream(stream)))
    return Wp2, sw2


@dataclass
class OutlierKernel:
    """Device buffers of an outlier-compensated uint8 kernel of a K x N
    weight (layouts of include/qlora.h, qlora_outlier_kernel)."""

    K: int
    N: int
    codes_nk: torch.Tensor  # [N, K] uint8
    codes_kn: torch.Tensor  # [K, N] uint8
    par: torch.Tensor       # [4] fp32: lo, hi, scale, bias
    start_nk: torch.Tensor  # [N * ceil(K/128) + 1] int32
    ent_nk: torch.Tensor    # [cap] int32 (uint32 entries)
    start_kn: torch.Tensor  # [K * ceil(N/128) + 1] int32
    ent_kn: torch.Tensor    # [cap] int32

    def struct(self) -> OutlierKernelStruct:
        return OutlierKernelStruct(self.codes_nk.data_ptr(), self.codes_kn.data_ptr(),
                                   self.par.data_ptr(), self.start_nk.data_ptr(),
                                   self.ent_nk.data_ptr(), self.start_kn.data_ptr(),
                                   self.ent_kn.data_ptr(), int(self.ent_nk.numel()))

    @property
    def count(self) -> int:
        """Number of outliers (reads the device tables)."""
        return int(self.start_nk[-1].item())


def qlora_outlier_cap(K: int, N: int) -> int:
    return int(_lib.qlora_outlier_cap(int(K), int(N)))


def qlora_outlier_workspace_bytes(K: int, N: int) -> int:
    return int(_lib.qlora_outlier_workspace_bytes(int(K), int(N)))


def outlier_kernel_buffers(K: int, N: int, device=None) -> OutlierKernel:
    dev = device or "cuda"
    cap = max(qlora_outlier_cap(K, N), 1)
    nbk, nbn = (K + 127) // 128, (N + 127) // 128
    return OutlierKernel(
        K, N, torch.empty((N, K), dtype=torch.uint8, device=dev),
        torch.empty((K, N), dtype=torch.uint8, device=dev),
        torch.empty((4,), dtype=torch.float32, device=dev),
        torch.empty((N * nbk + 1,), dtype=torch.int32, device=dev),
        torch.empty((cap,), dtype=torch.int32, device=dev),
        torch.empty((K * nbn + 1,), dtype=torch.int32, device=dev),
        torch.empty((cap,), dtype=torch.int32, device=dev))


def qlora_outlier_quantize(W: torch.Tensor, q: OutlierKernel, ws: torch.Tensor, stream=None):
    K, N = W.shape
    assert W.dtype == torch.float32 and (q.K, q.N) == (K, N)
    st = q.struct()
    _check(_lib.qlora_outlier_quantize(_ptr(W), K, N, ctypes.byref(st), _ptr(ws), ws.numel(),
                                       _stream(stream)))


def quantize_outlier(W: torch.Tensor, stream=None) -> OutlierKernel:
    """W [K, N] fp32 -> its outlier-compensated kernel (fresh buffers)."""
    K, N = W.shape
    W = W.float().contiguous()
    q = outlier_kernel_buffers(K, N, W.device)
    ws = torch.empty(qlora_outlier_workspace_bytes(K, N), dtype=torch.uint8, device=W.device)
    qlora_outlier_quantize(W, q, ws, stream)
    return q


def qlora_outlier_forward(d: LayerDesc, M: int, X, q: OutlierKernel, bias, A, B, Y, xA, ws,
                          stream=None):
    st = q.struct()
    _check(_lib.qlora_outlier_forward(ctypes.byref(d), int(M), _ptr(X), ctypes.byref(st), _ptr(bias),
                                      _ptr(A), _ptr(B), _ptr(Y), _ptr(xA), _ptr(ws), ws.numel(),
                                      _stream(stream)))


def qlora_outlier_backward(d: LayerDesc, M: int, X, dY, q: OutlierKernel, A, B, xA, dX, dA, dB,
                           dbias, ws, stream=None):
    st = q.struct()
    _check(_lib.qlora_outlier_backward(ctypes.byref(d), int(M), _ptr(X), _ptr(dY), ctypes.byref(st),
                                       _ptr(A), _ptr(B), _ptr(xA), _ptr(dX), _ptr(dA), _ptr(dB),
                                       _ptr(dbias), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_permute(src: torch.Tensor, perm, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dst = src with its axes permuted (dst axis d is src axis perm[d]), by
    the library's kernel; returns dst (contiguous)."""
    perm = [int(p) for p in perm]
    nd = src.dim()
    if sorted(perm) != list(range(nd)):
        raise ValueError("perm must be a permutation of 0 .. %d" % (nd - 1))
    shape = [src.shape[p] for p in perm]
    dst = out if out is not None else torch.empty(shape, dtype=src.dtype, device=src.device)
    if tuple(dst.shape) != tuple(shape) or dst.dtype != src.dtype:
        raise ValueError("out has the wrong shape or dtype")
    if src.numel() == 0:
        return dst
    sh = (ctypes.c_int64 * nd)(*src.shape)
    pm = (ctypes.c_int * nd)(*perm)
    _check(_lib.qlora_permute(_ptr(src), _ptr(dst), nd, sh, pm, src.element_size(), _stream(stream)))
    return dst


FP8_E4M3 = 0
FP8_E5M2 = 1
FP8_WORKSPACE_BYTES = 256


def qlora_fp8_quantize(T: torch.Tensor, fmt: int, scale_in, scale_out, history, q, qt=None, ws=None,
                       stream=None):
    """Codes of T [rows, cols] with *scale_in into q (and its transpose into
    qt), then the next scale into scale_out and the rolled amax history."""
    rows, cols = T.shape
    if ws is None:
        ws = torch.empty(FP8_WORKSPACE_BYTES, dtype=torch.uint8, device=T.device)
    _check(_lib.qlora_fp8_quantize(_ptr(T), rows, cols, act_code(T.dtype), int(fmt), _ptr(scale_in),
                                   _ptr(scale_out), _ptr(history), history.numel(), _ptr(q), _ptr(qt),
                                   _ptr(ws), ws.numel(), _stream(stream)))


def qlora_fp8_colsum_workspace_bytes(rows: int, cols: int) -> int:
    return int(_lib.qlora_fp8_colsum_workspace_bytes(int(rows), int(cols)))


def fp8_colsum_applies(T: torch.Tensor, q: torch.Tensor, qt=None) -> bool:
    """Whether qlora_fp8_quantize_colsum takes these tensors (its layout
    condition, checked here so a caller can choose another route)."""
    rows, cols = T.shape
    ok = T.data_ptr() % 16 == 0 and cols % 8 == 0 and q.data_ptr() % 8 == 0
    if qt is not None:
        ok = ok and qt.data_ptr() % 16 == 0 and rows % 16 == 0
    return bool(ok)


def qlora_fp8_quantize_colsum(T: torch.Tensor, fmt: int, scale_in, scale_out, history, q, qt, colsum, ws,
                              stream=None):
    """qlora_fp8_quantize plus colsum [cols] = column sums of T (fp32), in
    the same pass; ws: qlora_fp8_colsum_workspace_bytes(rows, cols) bytes."""
    rows, cols = T.shape
    _check(_lib.qlora_fp8_quantize_colsum(_ptr(T), rows, cols, act_code(T.dtype), int(fmt), _ptr(scale_in),
                                          _ptr(scale_out), _ptr(history), history.numel(), _ptr(q), _ptr(qt),
                                          _ptr(colsum), _ptr(ws), ws.numel(), _stream(stream)))


def qlora_fp8_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.qlora_fp8_gemm_workspace_bytes(int(M), int(N), int(K)))


def qlora_fp8_gemm_ws(A, fmt_a: int, B, fmt_b: int, scale_a, scale_b, bias, C, ws, stream=None):
    """qlora_fp8_gemm with a workspace for splitting a partial last wave of
    CTA-pair tiles (ws may be None: no split)."""
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and tuple(C.shape) == (M, N)
    _check(_lib.qlora_fp8_gemm_ws(_ptr(A), int(fmt_a), _ptr(B), int(fmt_b), M, N, K, _ptr(scale_a),
                                  _ptr(scale_b), _ptr(bias), _ptr(C), act_code(C.dtype), _ptr(ws),
                                  ws.numel() if ws is not None else 0, _stream(stream)))


def qlora_fp8_gemm(A, fmt_a: int, B, fmt_b: int, scale_a, scale_b, bias, C, stream=None):
    """C [M,N] = (A [M,K] B [N,K]^T) * scale_a * scale_b (+ bias)."""
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and tuple(C.shape) == (M, N)
    _check(_lib.qlora_fp8_gemm(_ptr(A), int(fmt_a), _ptr(B), int(fmt_b), M, N, K, _ptr(scale_a),
                               _ptr(scale_b), _ptr(bias), _ptr(C), act_code(C.dtype), _stream(stream)))


def qlora_set_rank_pass_rows(rows: int) -> int:
    """Minimum rows per CTA of the dB/dbias and dA passes (0: the default,
    lowest-latency spread); returns the previous setting."""
    prev = _lib.qlora_set_rank_pass_rows(int(rows))
    if prev < 0:
        _check(prev)
    return prev


def qlora_relu(Y: torch.Tensor, stream=None):
    _check(_lib.qlora_relu(_ptr(Y), Y.numel(), act_code(Y.dtype), _stream(stream)))


def qlora_relu_backward(dY: torch.Tensor, Y: torch.Tensor, stream=None):
    assert dY.shape == Y.shape and dY.dtype == Y.dtype
    _check(_lib.qlora_relu_backward(_ptr(dY), _ptr(Y), Y.numel(), act_code(Y.dtype), _stream(stream)))


def qlora_selftest_wait_timeout(limit_us: int, stream=None):
    _check(_lib.qlora_selftest_wait_timeout(int(limit_us), _stream(stream)))


def qlora_device_status(stream=None) -> int:
    return int(_lib.qlora_device_status(_stream(stream)))


@dataclass
class Layer:
    """Device buffers of one int8-LoRA Dense layer (frozen Wq/sw, trainable A/B)."""

    Wq: torch.Tensor
    sw: torch.Tensor
    bias: Optional[torch.Tensor]
    A: torch.Tensor
    B: torch.Tensor
    alpha: float
    act: torch.dtype

    @property
    def K(self):
        return self.Wq.shape[1]

    @property
    def N(self):
        return self.Wq.shape[0]

    @property
    def r(self):
        return self.A.shape[1]

    def desc(self) -> LayerDesc:
        return desc(self.K, self.N, self.r, self.alpha, self.act)


def forward(layer: Layer, X: torch.Tensor, ws: torch.Tensor, Y=None, xA=None, debug: bool = False,
            stream=None):
    """Returns (Y, xA[, (Xq, sx, acc)])."""
    M = X.shape[0]
    dev = X.device
    Y = Y if Y is not None else torch.empty((M, layer.N), dtype=layer.act, device=dev)
    xA = xA if xA is not None else torch.empty((M, layer.r), dtype=torch.float32, device=dev)
    dbg = None
    if debug:
        xq = torch.empty((M, layer.K), dtype=torch.int8, device=dev)
        sx = torch.empty((M,), dtype=torch.float32, device=dev)
        acc = torch.empty((M, layer.N), dtype=torch.int32, device=dev)
        dbg = Debug(xq.data_ptr(), sx.data_ptr(), acc.data_ptr())
    qlora_forward(layer.desc(), M, X, layer.Wq, layer.sw, layer.bias, layer.A, layer.B, Y, xA, ws,
                  dbg, stream)
    if debug:
        return Y, xA, (xq, sx, acc)
    return Y, xA


def backward(layer: Layer, X, dY, xA, ws, dX=None, want_dx=True, want_dbias=True, stream=None):
    """Returns (dX or None, dA, dB, dbias or None)."""
    M = X.shape[0]
    dev = X.device
    if want_dx and dX is None:
        dX = torch.empty((M, layer.K), dtype=layer.act, device=dev)
    dA = torch.empty((layer.K, layer.r), dtype=torch.float32, device=dev)
    dB = torch.empty((layer.r, layer.N), dtype=torch.float32, device=dev)
    dbias = torch.empty((layer.N,), dtype=torch.float32, device=dev) if want_dbias else None
    qlora_backward(layer.desc(), M, X, dY, layer.Wq, layer.sw, layer.A, layer.B, xA,
                   dX if want_dx else None, dA, dB, dbias, ws, stream)
    return (dX if want_dx else None), dA, dB, dbias


def merge(layer: Layer, stream=None):
    Wq2 = torch.empty_like(layer.Wq)
    sw2 = torch.empty_like(layer.sw)
    qlora_merge(layer.desc(), layer.Wq, layer.sw, layer.A, layer.B, Wq2, sw2, stream)
    return Wq2, sw2
