"""Blockwise 4-bit formats that the pages compare with NF4 + double quantisation.

TEST INFRASTRUCTURE ONLY, under the same rule as the rest of ``oracle/``: only the tests,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` may import it.

Sources:
* Page "QLoRA: put the large model in memory, then change it with a small adapter"
  (wq-win.github.io/llm/074-qlora), section 4, evidence 1. It quotes the paper's Table 2, which
  ranks four 4-bit formats by mean perplexity: Int4, FP4 E2M1, FP4 E3M0 and NF4 + DQ.
* Page "QLoRA" (weimeta.cn glossary), the paragraph on what NF4 4-bit quantisation is. It
  claims a 2 to 3 times smaller error than plain INT4 at the same width.

The pages name the formats but print neither their value sets nor their scaling. The readings
below are the plainest ones:
* Every format quantises 64-weight blocks, each scaled by the block's absmax c. c is kept in
  fp32 and is not double-quantised. |w| = c maps to the format's largest magnitude S.
* Int4: the 15 symmetric integers -7..7, S = 7.
* FP4 E2M1: a sign, 2 exponent bits (bias 1) and 1 mantissa bit, with subnormals. The
  magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6, so S = 6.
* FP4 E3M0: a sign and 3 exponent bits, no mantissa. Exponent field 0 means zero. The largest
  code maps to 1, so the magnitudes are 0 and 2^(e-7) for e = 1..7, S = 1.
* x' = fl(fl(w / c) * S) in fp32. The magnitude index is the number of decision thresholds
  (midpoints of consecutive magnitudes) strictly below |x'|. A tie, where |x'| sits exactly on
  a midpoint, goes to the even index. The sign is a separate bit, and -0 folds to +0.
* The dequantised weight is bf16(fl(v * fl(c / S))), with v the signed magnitude. This is the
  same bf16 output as the NF4 path's bf16(fl(Q * c^)).
An all-zero block (c = 0) gives zero codes and zero weights.

The magnitude tables are written out from those definitions. The tests derive them again from
the bit fields and pin the quantiser against a brute-force nearest search.
"""
from __future__ import annotations

import numpy as np

BLOCK = 64

# largest-magnitude units S and the eight magnitudes of each format (index 0..7)
FORMATS = {
    "int4": (7.0, [0.0, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0]),
    "fp4_e2m1": (6.0, [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]),
    "fp4_e3m0": (1.0, [0.0, 2.0 ** -6, 2.0 ** -5, 2.0 ** -4, 2.0 ** -3, 2.0 ** -2, 2.0 ** -1, 1.0]),
}


def magnitudes(fmt: str) -> np.ndarray:
    return np.array(FORMATS[fmt][1], dtype=np.float32)


def thresholds(fmt: str) -> np.ndarray:
    """Midpoints of consecutive magnitudes (exact in fp32 for all three formats)."""
    m = np.array(FORMATS[fmt][1], dtype=np.float64)
    t = (m[:-1] + m[1:]) / 2.0
    assert np.array_equal(t.astype(np.float32).astype(np.float64), t)
    return t.astype(np.float32)


def bf16_rne(f: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of finite fp32 values, round to nearest even."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def block_absmax(w: np.ndarray) -> np.ndarray:
    """c per 64-block of a flat fp32 array (a ragged last block uses its own elements)."""
    w = np.ascontiguousarray(w, dtype=np.float32).ravel()
    nb = -(-w.size // BLOCK)
    pad = np.zeros(nb * BLOCK, dtype=np.float32)
    pad[: w.size] = np.abs(w)
    return pad.reshape(nb, BLOCK).max(axis=1)


def quantize(w: np.ndarray, fmt: str):
    """(codes, c): codes uint8 per weight (bit 3 = sign, bits 0-2 = magnitude index), c fp32 per block."""
    S, _ = FORMATS[fmt]
    w = np.ascontiguousarray(w, dtype=np.float32).ravel()
    c = block_absmax(w)
    cw = np.repeat(c, BLOCK)[: w.size]
    with np.errstate(invalid="ignore", divide="ignore"):
        x = np.where(cw > 0, (w / cw).astype(np.float32) * np.float32(S), np.float32(0.0)).astype(np.float32)
    m = np.abs(x)
    T = thresholds(fmt)
    idx = np.searchsorted(T, m, side="left")           # number of thresholds strictly below m
    on_mid = (idx < T.size) & (m == T[np.minimum(idx, T.size - 1)])
    idx = np.where(on_mid & (idx % 2 == 1), idx + 1, idx)
    neg = (x < 0) & (idx > 0)
    codes = (idx | (neg.astype(np.int64) << 3)).astype(np.uint8)
    return codes, c


def dequant(codes: np.ndarray, c: np.ndarray, fmt: str) -> np.ndarray:
    """bf16 bit patterns of the dequantised weights."""
    S, _ = FORMATS[fmt]
    codes = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
    mag = magnitudes(fmt)[codes & 7]
    v = np.where(codes & 8, -mag, mag).astype(np.float32)
    step = (np.ascontiguousarray(c, dtype=np.float32) / np.float32(S)).astype(np.float32)
    cw = np.repeat(step, BLOCK)[: codes.size]
    return bf16_rne((v * cw).astype(np.float32))


def error_stats(w: np.ndarray, w_hat_bits: np.ndarray) -> dict:
    """Mean squared error, its ratio to the mean square of w, and the SNR in dB, in fp64."""
    w64 = np.ascontiguousarray(w, dtype=np.float32).ravel().astype(np.float64)
    h = (np.ascontiguousarray(w_hat_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    e = w64 - h.astype(np.float64)
    se, sw = float(np.dot(e, e)), float(np.dot(w64, w64))
    return {"mse": se / w64.size, "nmse": se / sw if sw > 0 else 0.0,
            "snr_db": 10.0 * np.log10(sw / se) if se > 0 else float("inf")}
