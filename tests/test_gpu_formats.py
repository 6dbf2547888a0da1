"""GPU parity of the Int4 / FP4 E2M1 / FP4 E3M0 reference formats (qlora_fmt4_quantize,
qlora_fmt4_dequant) against the oracle (oracle/formats.py): block constants, packed codes and
the bf16 dequantised weights, all bit for bit."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import oracle
from oracle import formats as F

pytestmark = pytest.mark.gpu

FMTS = ("int4", "fp4_e2m1", "fp4_e3m0")


def pack(codes):
    c = np.asarray(codes, dtype=np.uint8)
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, dtype=np.uint8)])
    return (c[0::2] << 4) | c[1::2]


def tie_values(fmt, c):
    """Weights whose normalised value x' = fl(fl(w / c) * S) is exactly a midpoint."""
    S = F.FORMATS[fmt][0]
    out = []
    for t in F.thresholds(fmt):
        w = np.float32(float(t) * float(c) / S)
        for _ in range(8):
            x = (np.float32(w) / np.float32(c)).astype(np.float32) * np.float32(S)
            if x == t:
                out.append(w)
                break
            w = np.nextafter(w, np.float32(np.inf) if x < t else np.float32(-np.inf))
    return np.array(out, dtype=np.float32)


def make_input(n, fmt, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    if n >= 256:
        w[64:128] = 0.0                                   # an all-zero block
        w[rng.choice(n, max(1, n // 1000), replace=False)] *= 10.0
        t = tie_values(fmt, 0.75)
        w[128:192] *= 0.01                                # block 2: absmax 0.75 and exact ties
        w[128] = 0.75
        w[129:129 + t.size] = t
        w[160:160 + t.size] = -t
        w[191] = -0.75
    return w


def check(w_np, W_dev, fmt):
    n = w_np.size
    codes, absmax = q.qlora_fmt4_quantize(W_dev, fmt)
    out = q.qlora_fmt4_dequant(codes, absmax, n, fmt)
    assert q.qlora_get_device_status() == q.QLORA_OK
    ref_codes, ref_c = F.quantize(w_np, fmt)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), ref_c.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), pack(ref_codes))
    ref = F.dequant(ref_codes, ref_c, fmt)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n", [1, 63, 64 * 7 + 13, 64 * 64, 1 << 20])
def test_fp32_input_bit_exact(fmt, n):
    w = make_input(n, fmt, seed=n + len(fmt))
    check(w, torch.from_numpy(w).cuda(), fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_bf16_input_bit_exact(fmt):
    w = make_input(64 * 300 + 31, fmt, seed=77)
    W = torch.from_numpy(w).to(torch.bfloat16).cuda()
    # the oracle sees the exact fp32 widening of the bf16 values
    check(W.float().cpu().numpy(), W, fmt)


def test_gaussian_error_matches_oracle():
    # the error statistics the oracle comparison reports, from the device's dequantised weights
    rng = np.random.default_rng(2024)
    w = (rng.standard_normal(1 << 18) * 0.02).astype(np.float32)
    W = torch.from_numpy(w).cuda()
    for fmt in FMTS:
        codes, absmax = q.qlora_fmt4_quantize(W, fmt)
        out = q.qlora_fmt4_dequant(codes, absmax, w.size, fmt)
        got = F.error_stats(w, out.view(torch.int16).cpu().numpy().view(np.uint16))
        rc, cc = F.quantize(w, fmt)
        ref = F.error_stats(w, F.dequant(rc, cc, fmt))
        assert got == ref
