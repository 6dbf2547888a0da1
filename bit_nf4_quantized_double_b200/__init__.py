"""Python binding of libqlora_nf4.so (the QLoRA NF4 + double-quant layer, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/qlora_nf4.h. PyTorch supplies
device memory and streams. There is no fallback: if the shared library is
missing, importing the binding's entry points raises.

Entry points (same names as the C ABI):
    qlora_nf4_quantize(W)                    -> NF4Tensor
    qlora_nf4_dequant(q)                     -> bf16 [rows, cols]
    qlora_linear_fwd(X, q, A, B, s)          -> (Y, XA)
    qlora_linear_bwd(X, dY, q, A, B, s, XA)  -> (dX, dA, dB)
    qlora_get_device_status()                -> status code (0 = ok)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = 1
QLORA_ERR_UNSUPPORTED_SHAPE = 2
QLORA_ERR_WORKSPACE = 3
QLORA_ERR_NONFINITE = 4
QLORA_ERR_TIMEOUT = 5
QLORA_ERR_CUDA = 6
QLORA_F32 = 0
QLORA_BF16 = 1


class QloraError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: status {status} ({status_string(status)})")


class _Tensor(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("scale8", ctypes.c_void_p), ("scale2", ctypes.c_void_p), ("offset", ctypes.c_void_p)]


_lib = None

class _LinearDesc(ctypes.Structure):
    """qlora_linear_desc of the C ABI."""
    _fields_ = [("X", ctypes.c_void_p), ("W", ctypes.POINTER(_Tensor)), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("r", ctypes.c_int), ("s", ctypes.c_float), ("Y", ctypes.c_void_p),
                ("XA_save", ctypes.c_void_p)]


_SIGS = {
    "qlora_nf4_storage_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "qlora_nf4_quantize_workspace": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "qlora_nf4_quantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(_Tensor), ctypes.c_void_p,
                                          ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_nf4_dequant": (ctypes.c_int, [ctypes.POINTER(_Tensor), ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_linear_fwd_workspace": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "qlora_linear_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(_Tensor), ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_bwd_workspace": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "qlora_linear_bwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(_Tensor),
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_fwd_grouped_workspace": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int,
                                                            ctypes.POINTER(_LinearDesc)]),
    "qlora_linear_fwd_grouped": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(_LinearDesc),
                                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_nf4_quantize_grouped_workspace": (ctypes.c_size_t, [ctypes.c_int, ctypes.POINTER(_Tensor)]),
    "qlora_nf4_quantize_grouped": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int,
                                                  ctypes.POINTER(_Tensor), ctypes.c_void_p, ctypes.c_size_t,
                                                  ctypes.c_void_p]),
    "qlora_nf4_dequant_grouped": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(_Tensor),
                                                 ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p]),
    "qlora_nf4_set_code_search": (None, [ctypes.c_int]),
    "qlora_linear_set_pair_min_m": (None, [ctypes.c_int64]),
    "qlora_adamw_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_adamw_prefetch": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]),
    "qlora_get_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_nf4_codebook": (None, [ctypes.c_void_p]),
    "qlora_nf4_quantize_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(_Tensor),
                                                  ctypes.c_void_p]),
    "qlora_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_void_p]),
    "qlora_selftest_rcp_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_nf4_merge_workspace": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "qlora_nf4_merge_adapter": (ctypes.c_int, [ctypes.POINTER(_Tensor), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_float, ctypes.c_void_p, ctypes.POINTER(_Tensor),
                                               ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_fmt4_quantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_fmt4_dequant": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_launch_count": (ctypes.c_ulonglong, []),
    "qlora_profile_enable": (None, [ctypes.c_int]),
    "qlora_profile_read": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                          ctypes.POINTER(ctypes.c_int)]),
}


def lib() -> ctypes.CDLL:
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not found: build it with bit_nf4_quantized_double_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().qlora_status_string(int(s)).decode()


def _check(status: int, what: str):
    if status != QLORA_OK:
        raise QloraError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _hold(stream, *tensors):
    """Temporaries made for a call (contiguous copies, a workspace) are freed when the
    wrapper returns, while the kernels queued on `stream` may still read them. torch's
    caching allocator only orders reuse on the current stream, so when the call went
    to another stream the blocks are marked as in use by that stream as well."""
    if stream is None or stream == torch.cuda.current_stream():
        return
    for t in tensors:
        if t is not None:
            t.record_stream(stream)


@dataclass
class NF4Tensor:
    """The stored format: four device buffers owned by torch."""
    rows: int
    cols: int
    codes: torch.Tensor    # uint8 [ceil(n/2)]
    scale8: torch.Tensor   # int8 [ceil(n/64)]
    scale2: torch.Tensor   # float32 [ceil(nb/256)]
    offset: torch.Tensor   # float32 [1]

    def ctype(self) -> _Tensor:
        return _Tensor(self.rows, self.cols, self.codes.data_ptr(), self.scale8.data_ptr(),
                       self.scale2.data_ptr(), self.offset.data_ptr())

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.scale8, self.scale2, self.offset))


def nf4_sizes(rows: int, cols: int):
    n = rows * cols
    nb = -(-n // 64)
    return n, -(-n // 2), nb, -(-nb // 256)


def nf4_empty(rows: int, cols: int, device="cuda") -> NF4Tensor:
    n, ncode, nb, nb2 = nf4_sizes(rows, cols)
    return NF4Tensor(rows, cols, torch.empty(ncode, dtype=torch.uint8, device=device),
                     torch.empty(nb, dtype=torch.int8, device=device),
                     torch.empty(nb2, dtype=torch.float32, device=device),
                     torch.empty(1, dtype=torch.float32, device=device))


def _workspace(nbytes: int, device, ws=None):
    if nbytes == 0:
        return None, 0
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws, ws.numel() * ws.element_size()
    t = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return t, nbytes


def qlora_nf4_storage_bytes(rows: int, cols: int) -> int:
    return int(lib().qlora_nf4_storage_bytes(rows, cols))


def qlora_nf4_codebook():
    buf = (ctypes.c_float * 16)()
    lib().qlora_nf4_codebook(ctypes.cast(buf, ctypes.c_void_p))
    return [float(v) for v in buf]


def qlora_nf4_quantize(W: torch.Tensor, out: NF4Tensor | None = None, ws: torch.Tensor | None = None,
                       stream=None) -> NF4Tensor:
    """Quantise a [rows, cols] fp32 or bf16 CUDA tensor (contiguous)."""
    if W.dim() == 1:
        W = W.view(1, -1)
    rows, cols = W.shape
    dt = {torch.float32: QLORA_F32, torch.bfloat16: QLORA_BF16}[W.dtype]
    if out is None:
        out = nf4_empty(rows, cols, W.device)
    L = lib()
    need = int(L.qlora_nf4_quantize_workspace(rows, cols))
    wsb, wsn = _workspace(need, W.device, ws)
    t = out.ctype()
    Wc = W.contiguous()
    _check(L.qlora_nf4_quantize(_ptr(Wc), dt, ctypes.byref(t), _ptr(wsb), wsn, _stream(stream)),
           "qlora_nf4_quantize")
    _hold(stream, Wc, wsb)
    return out


def qlora_nf4_dequant(q: NF4Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=q.codes.device)
    t = q.ctype()
    _check(lib().qlora_nf4_dequant(ctypes.byref(t), _ptr(out), _stream(stream)), "qlora_nf4_dequant")
    return out


def qlora_nf4_quantize_grouped(Ws, outs=None, ws: torch.Tensor | None = None, stream=None):
    """Quantise a list of [rows, cols] CUDA tensors of one dtype (fp32 or bf16) with one
    sequence of launches. Returns the list of NF4Tensor."""
    Ws = [W.view(1, -1) if W.dim() == 1 else W.contiguous() for W in Ws]
    dt = {torch.float32: QLORA_F32, torch.bfloat16: QLORA_BF16}[Ws[0].dtype]
    if any(W.dtype != Ws[0].dtype for W in Ws):
        raise ValueError("qlora_nf4_quantize_grouped: all tensors must share one dtype")
    if outs is None:
        outs = [nf4_empty(W.shape[0], W.shape[1], W.device) for W in Ws]
    n = len(Ws)
    ts = (_Tensor * n)(*[o.ctype() for o in outs])
    ptrs = (ctypes.c_void_p * n)(*[W.data_ptr() for W in Ws])
    L = lib()
    wsb, wsn = _workspace(int(L.qlora_nf4_quantize_grouped_workspace(n, ts)), Ws[0].device, ws)
    _check(L.qlora_nf4_quantize_grouped(n, ptrs, dt, ts, _ptr(wsb), wsn, _stream(stream)),
           "qlora_nf4_quantize_grouped")
    _hold(stream, wsb, *Ws)
    return outs


def qlora_nf4_dequant_grouped(qs, outs=None, stream=None):
    """Dequantise a list of NF4Tensor to bf16 [rows, cols] with one launch per 64 tensors."""
    if outs is None:
        outs = [torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=t.codes.device) for t in qs]
    n = len(qs)
    ts = (_Tensor * n)(*[t.ctype() for t in qs])
    ptrs = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    _check(lib().qlora_nf4_dequant_grouped(n, ts, ptrs, _stream(stream)), "qlora_nf4_dequant_grouped")
    return outs


class AdamwHparams(ctypes.Structure):
    """qlora_adamw_hparams of the C ABI."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


def qlora_adamw_step(theta: torch.Tensor, grad: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: int,
                     lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                     weight_decay: float = 0.0, theta_bf16: torch.Tensor | None = None, stream=None):
    """One AdamW step in place on fp32 CUDA (or managed) tensors theta, m, v with gradient grad;
    theta_bf16, when given, receives bf16(theta)."""
    n = theta.numel()
    for t in (grad, m, v):
        assert t.numel() == n and t.dtype == torch.float32 and t.is_contiguous()
    h = AdamwHparams(lr, beta1, beta2, eps, weight_decay, int(step))
    _check(lib().qlora_adamw_step(_ptr(theta), _ptr(grad), _ptr(m), _ptr(v), n, ctypes.byref(h), _ptr(theta_bf16),
                                  _stream(stream)), "qlora_adamw_step")


def qlora_adamw_prefetch(t: torch.Tensor, to_device: bool = True, stream=None):
    """Move the managed pages of tensor t to the current GPU (or back to host memory)."""
    _check(lib().qlora_adamw_prefetch(_ptr(t), t.numel() * t.element_size(), 1 if to_device else 0, _stream(stream)),
           "qlora_adamw_prefetch")


class _Managed:
    """A block of CUDA managed (unified) memory exposed to torch through the CUDA array
    interface, freed when the last tensor viewing it is gone. Plumbing for paged optimizer
    state; the library itself never allocates."""
    _cudart = None

    def __init__(self, nbytes: int):
        if _Managed._cudart is None:
            torch.cuda.init()
            _Managed._cudart = ctypes.CDLL("libcudart.so.12")
        p = ctypes.c_void_p()
        if _Managed._cudart.cudaMallocManaged(ctypes.byref(p), ctypes.c_size_t(max(nbytes, 16)), 1) != 0:
            raise MemoryError("cudaMallocManaged failed")
        self.ptr, self.nbytes = p.value, nbytes

    def __del__(self):
        if self.ptr and _Managed._cudart is not None:
            _Managed._cudart.cudaFree(ctypes.c_void_p(self.ptr))
            self.ptr = None


def managed_empty(n: int, dtype=torch.float32) -> torch.Tensor:
    """A 1-D tensor of n elements in CUDA managed memory (pages move between host and GPU on
    demand, or by qlora_adamw_prefetch)."""
    esz = torch.empty(0, dtype=dtype).element_size()
    blk = _Managed(n * esz)
    typestr = {torch.float32: "<f4", torch.bfloat16: "<V2", torch.int8: "|i1", torch.uint8: "|u1"}[dtype]

    class _View:
        __cuda_array_interface__ = {"shape": (n,), "typestr": typestr if dtype != torch.bfloat16 else "<i2",
                                    "data": (blk.ptr, False), "version": 2}
    t = torch.as_tensor(_View(), device="cuda")
    if dtype == torch.bfloat16:
        t = t.view(torch.bfloat16)
    t._qlora_managed = blk            # the memory lives as long as the tensor
    return t


FMT4 = {"int4": 0, "fp4_e2m1": 1, "fp4_e3m0": 2}


def qlora_fmt4_quantize(W: torch.Tensor, fmt: str, stream=None):
    """Blockwise Int4 / FP4 E2M1 / FP4 E3M0 (64-weight absmax blocks) of a fp32 or bf16 tensor.
    Returns (codes uint8 [ceil(n/2)], two codes per byte; absmax fp32 [ceil(n/64)])."""
    W = W.contiguous()
    n = W.numel()
    dt = {torch.float32: QLORA_F32, torch.bfloat16: QLORA_BF16}[W.dtype]
    codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=W.device)
    absmax = torch.empty((n + 63) // 64, dtype=torch.float32, device=W.device)
    _check(lib().qlora_fmt4_quantize(_ptr(W), dt, n, FMT4[fmt], _ptr(codes), _ptr(absmax), _stream(stream)),
           "qlora_fmt4_quantize")
    _hold(stream, W)
    return codes, absmax


def qlora_fmt4_dequant(codes: torch.Tensor, absmax: torch.Tensor, n: int, fmt: str, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """bf16 [n] from the codes and block constants of qlora_fmt4_quantize."""
    if out is None:
        out = torch.empty(n, dtype=torch.bfloat16, device=codes.device)
    _check(lib().qlora_fmt4_dequant(_ptr(codes), _ptr(absmax), n, FMT4[fmt], _ptr(out), _stream(stream)),
           "qlora_fmt4_dequant")
    return out


def qlora_linear_fwd(X: torch.Tensor, W: NF4Tensor, A: torch.Tensor | None, B: torch.Tensor | None, s: float,
                     Y: torch.Tensor | None = None, XA_save: torch.Tensor | bool | None = True,
                     ws: torch.Tensor | None = None, stream=None):
    """Y = X W^ + s (X A) B. Returns (Y, XA) where XA is bf16 [M, r] (or None)."""
    M = X.shape[0]
    r = 0 if A is None else A.shape[1]
    if Y is None:
        Y = torch.empty(M, W.rows, dtype=torch.bfloat16, device=X.device)
    if XA_save is True:
        XA_save = torch.empty(M, r, dtype=torch.bfloat16, device=X.device) if r else None
    elif XA_save is False:
        XA_save = None
    L = lib()
    wsb, wsn = _workspace(int(L.qlora_linear_fwd_workspace(M, W.rows, W.cols, r)), X.device, ws)
    t = W.ctype()
    _check(L.qlora_linear_fwd(_ptr(X), M, ctypes.byref(t), _ptr(A), _ptr(B), r, float(s), _ptr(Y),
                              _ptr(XA_save), _ptr(wsb), wsn, _stream(stream)), "qlora_linear_fwd")
    _hold(stream, wsb)
    return Y, XA_save


def qlora_nf4_merge_adapter(W: NF4Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                            out: NF4Tensor | None = None, W_bf16: torch.Tensor | None = None,
                            ws: torch.Tensor | None = None, stream=None):
    """Merge the adapter into the weight in BF16 and re-quantise: returns (W_out, W_bf16)
    with W_bf16 = bf16(Dequant(W) + s (A B)^T) [rows, cols] and W_out its NF4 + DQ form."""
    if out is None:
        out = nf4_empty(W.rows, W.cols, W.codes.device)
    if W_bf16 is None:
        W_bf16 = torch.empty(W.rows, W.cols, dtype=torch.bfloat16, device=W.codes.device)
    L = lib()
    wsb, wsn = _workspace(int(L.qlora_nf4_merge_workspace(W.rows, W.cols)), W.codes.device, ws)
    t, to = W.ctype(), out.ctype()
    _check(L.qlora_nf4_merge_adapter(ctypes.byref(t), _ptr(A), _ptr(B), A.shape[1], float(s), _ptr(W_bf16),
                                     ctypes.byref(to), _ptr(wsb), wsn, _stream(stream)), "qlora_nf4_merge_adapter")
    _hold(stream, wsb)
    return out, W_bf16


def qlora_linear_fwd_grouped(items, ws: torch.Tensor | None = None, stream=None):
    """Forward of several projections in one call (all with the same M).

    items: sequence of dicts with keys X, W (NF4Tensor), A, B (or None), s, and
    optionally Y (output) and XA_save (tensor, or None). Returns the list of Y."""
    items = list(items)
    M = items[0]["X"].shape[0]
    n = len(items)
    tensors = [it["W"].ctype() for it in items]          # kept alive for the call
    descs = (_LinearDesc * n)()
    outs = []
    for i, it in enumerate(items):
        X, W, A, B = it["X"], it["W"], it.get("A"), it.get("B")
        r = 0 if A is None else A.shape[1]
        Y = it.get("Y")
        if Y is None:
            Y = torch.empty(M, W.rows, dtype=torch.bfloat16, device=X.device)
        outs.append(Y)
        descs[i] = _LinearDesc(_ptr(X), ctypes.pointer(tensors[i]), _ptr(A), _ptr(B), r, float(it["s"]), _ptr(Y),
                               _ptr(it.get("XA_save")))
    L = lib()
    wsb, wsn = _workspace(int(L.qlora_linear_fwd_grouped_workspace(M, n, descs)), items[0]["X"].device, ws)
    _check(L.qlora_linear_fwd_grouped(M, n, descs, _ptr(wsb), wsn, _stream(stream)), "qlora_linear_fwd_grouped")
    _hold(stream, wsb)
    return outs


def qlora_linear_bwd(X: torch.Tensor, dY: torch.Tensor, W: NF4Tensor, A: torch.Tensor | None,
                     B: torch.Tensor | None, s: float, XA: torch.Tensor | None = None,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, stream=None):
    """dX = dY W^T + s (dY B^T) A^T, dA = s X^T (dY B^T), dB = s (XA)^T dY. Returns (dX, dA, dB)."""
    M = dY.shape[0]
    r = 0 if A is None else A.shape[1]
    dev = dY.device
    if dX is None:
        dX = torch.empty(M, W.cols, dtype=torch.bfloat16, device=dev)
    if r and dA is None:
        dA = torch.empty(W.cols, r, dtype=torch.float32, device=dev)
    if r and dB is None:
        dB = torch.empty(r, W.rows, dtype=torch.float32, device=dev)
    L = lib()
    wsb, wsn = _workspace(int(L.qlora_linear_bwd_workspace(M, W.rows, W.cols, r)), dev, ws)
    t = W.ctype()
    _check(L.qlora_linear_bwd(_ptr(X), _ptr(dY), M, ctypes.byref(t), _ptr(A), _ptr(B), r, float(s), _ptr(XA),
                              _ptr(dX), _ptr(dA), _ptr(dB), _ptr(wsb), wsn, _stream(stream)), "qlora_linear_bwd")
    _hold(stream, wsb)
    return dX, dA, dB


def qlora_get_device_status(stream=None) -> int:
    return int(lib().qlora_get_device_status(_stream(stream)))


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_profile_enable(on: bool = True) -> None:
    lib().qlora_profile_enable(1 if on else 0)


def qlora_profile_read(kernel: str | None = None):
    """(total milliseconds, launches) of the recorded launches of `kernel` (None: all)."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int(0)
    _check(lib().qlora_profile_read(kernel.encode() if kernel else None, ctypes.byref(ms), ctypes.byref(n)),
           "qlora_profile_read")
    return float(ms.value), int(n.value)
