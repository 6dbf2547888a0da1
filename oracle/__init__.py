"""CPU oracle for the QLoRA NF4 + double-quantisation linear layer.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import this package. The product
library never calls it, and it shares no code with the CUDA path.

What it computes, following "QLoRA: put the large model in memory, then
change it with a small adapter" (wq-win.github.io/llm/074-qlora):

* section 1, the layer equation: Y = X W^ + s X A B with W^ = Dequant(W4, scales);
  the frozen base gets no gradient but dX flows through W^ transposed;
* section 2, the storage format: 64-weight absmax blocks, a 16-value
  normal-quantile codebook with an exact zero, 8-bit first-level constants
  with an offset and one fp32 second-level constant per 256 constants;
* section 3, the order: quantise W, then quantise the first-level constants;
  dequantise to BF16 on demand.

The encoding steps run in ``nf4_oracle.c`` (plain C, one IEEE fp32 operation
per step, no FMA contraction). The products are the exact fp64 products of
the bf16 operands (numpy float64 matmul as a library primitive).

The stored weight uses the nn.Linear layout [d_out, d_in] (rows = d_out), so
the W^ of the layer equation is the transpose of the stored matrix.

Parity unpinned: the numeric codebook and the linear int8 map of the
first-level constants are readings of the pages (they print neither); only
invariants pin them, not a comparison with another NF4 implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

BLOCK1 = 64    # weights per first-level block (section 2)
BLOCK2 = 256   # first-level constants per second-level block (section 2)

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        L.orc_norm_quantile_upper.restype = ctypes.c_double
        L.orc_norm_quantile_upper.argtypes = [ctypes.c_double]
        L.orc_codebook_f64.argtypes = [ctypes.c_void_p]
        L.orc_codebook.argtypes = [ctypes.c_void_p]
        L.orc_midpoints.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        L.orc_code_of.restype = ctypes.c_int
        L.orc_code_of.argtypes = [ctypes.c_float, ctypes.c_void_p]
        L.orc_code_bruteforce.restype = ctypes.c_int
        L.orc_code_bruteforce.argtypes = [ctypes.c_float, ctypes.c_void_p]
        L.orc_sweep_codes.restype = ctypes.c_int64
        L.orc_sweep_codes.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int64)]
        L.orc_quantize_codes.restype = ctypes.c_int
        L.orc_quantize_codes.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_void_p]
        L.orc_pairwise_sum_f64.restype = ctypes.c_double
        L.orc_pairwise_sum_f64.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_offset.restype = ctypes.c_float
        L.orc_offset.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_double_quant.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_float,
                                       ctypes.c_void_p, ctypes.c_void_p]
        L.orc_dequant_constant.restype = ctypes.c_float
        L.orc_dequant_constant.argtypes = [ctypes.c_int8, ctypes.c_float, ctypes.c_float]
        L.orc_merge_bf16.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
        L.orc_merge_bf16.restype = None
        L.orc_dequant.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne.argtypes = [ctypes.c_float]
        L.orc_bf16_array_to_f32.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_max_threads.restype = ctypes.c_int
        L.orc_adamw_step.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int64] + [ctypes.c_float] * 7 + [ctypes.c_void_p]
        L.orc_adamw_bias_corrections.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_int64,
                                                 ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
        del f32p
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def threads() -> int:
    """Threads the oracle's OpenMP loops use (the count of host cores in play)."""
    return int(lib().orc_max_threads())


# --------------------------------------------------------------------------
# Codebook
# --------------------------------------------------------------------------
def norm_quantile_upper(p: float) -> float:
    return float(lib().orc_norm_quantile_upper(float(p)))


def codebook_f64() -> np.ndarray:
    out = np.zeros(16, dtype=np.float64)
    lib().orc_codebook_f64(_ptr(out))
    return out


def codebook() -> np.ndarray:
    out = np.zeros(16, dtype=np.float32)
    lib().orc_codebook(_ptr(out))
    return out


def midpoints(Q: np.ndarray | None = None) -> np.ndarray:
    Q = codebook() if Q is None else np.ascontiguousarray(Q, dtype=np.float32)
    T = np.zeros(15, dtype=np.float32)
    lib().orc_midpoints(_ptr(Q), _ptr(T))
    return T


def code_of(x: float, T: np.ndarray) -> int:
    return int(lib().orc_code_of(ctypes.c_float(x), _ptr(np.ascontiguousarray(T, np.float32))))


def code_bruteforce(x: float, Q: np.ndarray) -> int:
    return int(lib().orc_code_bruteforce(ctypes.c_float(x), _ptr(np.ascontiguousarray(Q, np.float32))))


def sweep_codes(Q: np.ndarray | None = None):
    """Exhaustive fp32 sweep of [-1, 1]: (mismatches off-threshold, tested, on-threshold)."""
    Q = codebook() if Q is None else np.ascontiguousarray(Q, dtype=np.float32)
    tested = ctypes.c_int64(0)
    onthr = ctypes.c_int64(0)
    bad = lib().orc_sweep_codes(_ptr(Q), ctypes.byref(tested), ctypes.byref(onthr))
    return int(bad), int(tested.value), int(onthr.value)


# --------------------------------------------------------------------------
# bf16 helpers (bit patterns held in uint16)
# --------------------------------------------------------------------------
def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32).ravel()
    out = np.empty(f.size, dtype=np.uint16)
    L = lib()
    for i in range(f.size):
        out[i] = L.orc_bf16_rne(ctypes.c_float(float(f[i])))
    return out


# --------------------------------------------------------------------------
# The format
# --------------------------------------------------------------------------
@dataclass
class NF4Tensor:
    rows: int
    cols: int
    codes: np.ndarray    # uint8 [ceil(n/2)], byte k = code[2k] << 4 | code[2k+1]
    scale8: np.ndarray   # int8 [nb], nb = ceil(n/64)
    scale2: np.ndarray   # float32 [nb2], nb2 = ceil(nb/256)
    offset: np.float32   # mu, the mean of the first-level constants
    c1: np.ndarray       # float32 [nb], the exact first-level absmax (not stored in the format)
    status: int          # 0 ok, 1 non-finite input

    @property
    def n(self) -> int:
        return self.rows * self.cols


def sizes(rows: int, cols: int):
    """(n, code bytes, nb, nb2) of a [rows, cols] tensor (section 2 layout)."""
    n = rows * cols
    nb = -(-n // BLOCK1)
    nb2 = -(-nb // BLOCK2)
    return n, -(-n // 2), nb, nb2


def storage_bytes(rows: int, cols: int) -> int:
    """Bytes of the stored format: codes + int8 constants + fp32 second-level
    constants + the fp32 offset."""
    n, ncode, nb, nb2 = sizes(rows, cols)
    return ncode + nb + 4 * nb2 + 4


def quantize(w: np.ndarray, rows: int | None = None, cols: int | None = None) -> NF4Tensor:
    """NF4 + double quantisation of an fp32 array (section 2 and section 3:
    quantise the weights first with the exact absmax, then the constants)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    if rows is None:
        rows, cols = (w.shape if w.ndim == 2 else (1, w.size))
    n, ncode, nb, nb2 = sizes(rows, cols)
    assert w.size == n
    L = lib()
    Q = codebook()
    c1 = np.zeros(nb, dtype=np.float32)
    codes = np.zeros(ncode, dtype=np.uint8)
    status = L.orc_quantize_codes(_ptr(w.ravel()), n, _ptr(Q), _ptr(c1), _ptr(codes))
    scratch = np.zeros(2 * nb, dtype=np.float64)
    mu = np.float32(L.orc_offset(_ptr(c1), nb, _ptr(scratch)))
    scale8 = np.zeros(nb, dtype=np.int8)
    scale2 = np.zeros(nb2, dtype=np.float32)
    L.orc_double_quant(_ptr(c1), nb, ctypes.c_float(float(mu)), _ptr(scale8), _ptr(scale2))
    return NF4Tensor(rows, cols, codes, scale8, scale2, mu, c1, int(status))


def quantize_bf16(w_bits: np.ndarray, rows: int, cols: int) -> NF4Tensor:
    """Same as quantize() for bf16 input given as uint16 bit patterns
    (widened exactly to fp32 first)."""
    return quantize(bf16_bits_to_f32(w_bits), rows, cols)


def pairwise_sum_f64(v: np.ndarray) -> float:
    v = np.ascontiguousarray(v, dtype=np.float64)
    scratch = np.zeros(max(v.size, 1), dtype=np.float64)
    return float(lib().orc_pairwise_sum_f64(_ptr(v), v.size, _ptr(scratch)))


def offset(c1: np.ndarray) -> np.float32:
    c1 = np.ascontiguousarray(c1, dtype=np.float32)
    scratch = np.zeros(2 * c1.size, dtype=np.float64)
    return np.float32(lib().orc_offset(_ptr(c1), c1.size, _ptr(scratch)))


def dequant_constants(q: NF4Tensor) -> np.ndarray:
    """c^_b for every first-level block (step 7)."""
    L = lib()
    out = np.empty(q.scale8.size, dtype=np.float32)
    mu = ctypes.c_float(float(q.offset))
    for b in range(q.scale8.size):
        out[b] = L.orc_dequant_constant(ctypes.c_int8(int(q.scale8[b])),
                                        ctypes.c_float(float(q.scale2[b // BLOCK2])), mu)
    return out


def dequant(q: NF4Tensor) -> np.ndarray:
    """W^ as bf16 bit patterns, flattened row-major (step 8)."""
    out = np.zeros(q.n, dtype=np.uint16)
    lib().orc_dequant(_ptr(q.codes), _ptr(q.scale8), _ptr(q.scale2), ctypes.c_float(float(q.offset)),
                      q.n, _ptr(codebook()), _ptr(out))
    return out


def merge_bf16(w_hat_bits: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """Merged BF16 weight w' = bf16(w^ + fl(s * sum_j A[k,j] B[j,n])) (fused multiply-adds in
    increasing j), as bf16 bits [rows, cols]. w_hat_bits: bf16 bits [rows, cols] of the
    dequantised weight; A [cols, r], B [r, rows]: fp32 arrays holding bf16 values."""
    rows, cols = w_hat_bits.shape
    r = A.shape[1]
    w = np.ascontiguousarray(w_hat_bits, dtype=np.uint16)
    a = np.ascontiguousarray(A, dtype=np.float32)
    b = np.ascontiguousarray(B, dtype=np.float32)
    out = np.empty((rows, cols), dtype=np.uint16)
    lib().orc_merge_bf16(_ptr(w), _ptr(a), _ptr(b), rows, cols, r, ctypes.c_float(s), _ptr(out))
    return out


def unpack_codes(codes: np.ndarray, n: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(2 * codes.size, dtype=np.uint8)
    out[0::2] = codes >> 4
    out[1::2] = codes & 15
    return out[:n]


# --------------------------------------------------------------------------
# The layer (section 1 equation), exact fp64 products of bf16 operands.
#   stored weight Ws [d_out, d_in]; W^ of the equation = Ws^T
#   Y  = X Ws^T + s (X A) B
#   dX = dY Ws + s (dY B^T) A^T
#   dA = s X^T (dY B^T)
#   dB = s (X A)^T dY
# --------------------------------------------------------------------------
def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def linear_fwd(X, Ws, A, B, s: float):
    X, Ws, A, B = map(_f64, (X, Ws, A, B))
    return X @ Ws.T + s * ((X @ A) @ B)


def linear_bwd(X, dY, Ws, A, B, s: float):
    X, dY, Ws, A, B = map(_f64, (X, dY, Ws, A, B))
    G = dY @ B.T
    dX = dY @ Ws + s * (G @ A.T)
    dA, dB = adapter_grads(X, dY, A, B, s)
    return dX, dA, dB


def adapter_grads(X, dY, A, B, s: float):
    """dA = s X^T (dY B^T), dB = s (X A)^T dY (the adapter half of linear_bwd)."""
    X, dY, A, B = map(_f64, (X, dY, A, B))
    return s * (X.T @ (dY @ B.T)), s * ((X @ A).T @ dY)


def lora_param_count(d_in: int, d_out: int, r: int) -> int:
    """Trainable adapter parameters of one layer: A is [d_in, r], B is [r, d_out]."""
    return d_in * r + r * d_out


def rel_errors(got, ref):
    """(max|err| / max|ref|, ||err||_F / ||ref||_F) in fp64."""
    got = _f64(got)
    ref = _f64(ref)
    err = got - ref
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    fref = float(np.linalg.norm(ref))
    return (float(np.max(np.abs(err))) / mref if mref > 0 else float(np.max(np.abs(err), initial=0.0)),
            float(np.linalg.norm(err)) / fref if fref > 0 else float(np.linalg.norm(err)))


# --------------------------------------------------------------------------
# Paged AdamW of the adapter (section 3: "update LoRA with a paged optimizer";
# section 2: the optimizer state lives in unified memory). One step on fp32
# master parameters, fp32 moments; the operation order is in nf4_oracle.c.
# --------------------------------------------------------------------------
def adamw_bias_corrections(b1: float, b2: float, t: int):
    """Inverse bias corrections (1 / (1 - b1^t), 1 / (1 - b2^t)) in double, rounded once to fp32."""
    ib1, ib2 = ctypes.c_float(0.0), ctypes.c_float(0.0)
    lib().orc_adamw_bias_corrections(b1, b2, int(t), ctypes.byref(ib1), ctypes.byref(ib2))
    return np.float32(ib1.value), np.float32(ib2.value)


def adamw_step(theta: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, t: int, lr: float,
               b1: float = 0.9, b2: float = 0.999, eps: float = 1e-8, wd: float = 0.0, want_bf16: bool = False):
    """One AdamW step in place on fp32 arrays theta, m, v (gradient g). Returns bf16 bits of
    the new theta when want_bf16, else None."""
    for a in (theta, g, m, v):
        assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"]
    n = theta.size
    ib1, ib2 = adamw_bias_corrections(b1, b2, t)
    out = np.empty(n, dtype=np.uint16) if want_bf16 else None
    lib().orc_adamw_step(_ptr(theta), _ptr(g), _ptr(m), _ptr(v), n, lr, b1, b2, eps, wd, float(ib1), float(ib2),
                         _ptr(out) if want_bf16 else None)
    return out

