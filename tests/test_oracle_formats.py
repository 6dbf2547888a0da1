"""Pins of the oracle's Int4 / FP4 E2M1 / FP4 E3M0 blockwise formats (oracle/formats.py) and
the CPU comparison of their quantisation error with NF4 + double quantisation.

The pins do not re-type the oracle's formulas:
- the value sets are derived again from the sign / exponent / mantissa bit fields;
- the quantiser is checked against a brute-force nearest search over the signed values,
  on random inputs and on inputs built to land exactly on decision midpoints;
- the error is checked against the half-gap bound and, for the uniform Int4 grid, against
  the closed form step^2 / 12;
- the vectorised bf16 rounding is checked against the C oracle's scalar routine.
"""
import numpy as np
import pytest

import oracle
from oracle import formats as F

FMTS = ("int4", "fp4_e2m1", "fp4_e3m0")


def fp4_values(e_bits, m_bits, bias, subnormals):
    """Non-negative values of a sign/exponent/mantissa format with no inf/nan codes."""
    vals = set()
    for e in range(1 << e_bits):
        for m in range(1 << m_bits):
            frac = m / (1 << m_bits) if m_bits else 0.0
            if e == 0:
                vals.add(frac * 2.0 ** (1 - bias) if subnormals else 0.0)
            else:
                vals.add((1.0 + frac) * 2.0 ** (e - bias))
    return sorted(vals)


def test_value_sets_from_bit_fields():
    assert fp4_values(2, 1, 1, True) == list(F.magnitudes("fp4_e2m1"))
    # E3M0: exponent field 0 is zero, the largest exponent maps to 1 (bias 7)
    assert fp4_values(3, 0, 7, False) == list(F.magnitudes("fp4_e3m0"))
    assert list(F.magnitudes("int4")) == list(range(8))
    for f in FMTS:
        assert F.FORMATS[f][0] == F.magnitudes(f)[-1]


def normalised(w, c, S):
    """x' = fl(fl(w / c) * S) in fp32, as the readings define it."""
    return (np.float32(w) / np.float32(c)).astype(np.float32) * np.float32(S)


def brute_code(xp, fmt):
    mags = F.magnitudes(fmt).astype(np.float64)
    d = np.abs(abs(float(xp)) - mags)
    best = np.flatnonzero(d == d.min())
    i = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return i | (8 if (xp < 0 and i > 0) else 0)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_matches_bruteforce(fmt):
    S = F.FORMATS[fmt][0]
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(64 * 40) * 0.03).astype(np.float32)
    w[5] = 0.0
    w[70] = -0.0
    codes, c = F.quantize(w, fmt)
    for i in range(w.size):
        xp = normalised(w[i], c[i // 64], S)
        assert codes[i] == brute_code(xp, fmt), (i, w[i], xp)


@pytest.mark.parametrize("fmt", FMTS)
def test_ties_go_to_even_index(fmt):
    # inputs whose normalised value lands exactly on each midpoint
    S = F.FORMATS[fmt][0]
    T = F.thresholds(fmt)
    c = np.float32(0.75)
    hits = []
    for t in T:
        w0 = np.float32(float(t) * float(c) / S)
        for k in range(-4, 5):
            w = np.nextafter(w0, np.float32(np.inf) if k > 0 else np.float32(-np.inf)) if k else w0
            for _ in range(abs(k) - 1):
                w = np.nextafter(w, np.float32(np.inf) if k > 0 else np.float32(-np.inf))
            if normalised(w, c, S) == t:
                hits.append(w)
                break
    assert len(hits) >= len(T) - 2
    block = np.zeros(64, dtype=np.float32)
    block[0] = c
    block[1:1 + len(hits)] = hits
    block[20:20 + len(hits)] = -np.array(hits, dtype=np.float32)
    codes, cc = F.quantize(block, fmt)
    assert cc[0] == c
    for j, w in enumerate(hits):
        xp = normalised(w, c, S)
        i = int(np.searchsorted(T, abs(xp)))
        expect = i if i % 2 == 0 else i + 1
        assert codes[1 + j] == expect
        assert codes[20 + j] == (expect | 8 if expect else 0)
        assert codes[1 + j] == brute_code(xp, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_grid_values_round_trip(fmt):
    # c = S makes the quantisation step c / S exactly 1: every signed magnitude comes back exactly
    S = F.FORMATS[fmt][0]
    mags = F.magnitudes(fmt)
    vals = np.concatenate([mags, -mags[1:]]).astype(np.float32)
    block = np.zeros(64, dtype=np.float32)
    block[: vals.size] = vals
    codes, c = F.quantize(block, fmt)
    assert c[0] == np.float32(S)
    back = oracle.bf16_bits_to_f32(F.dequant(codes, c, fmt))
    assert np.array_equal(back[: vals.size], vals)


@pytest.mark.parametrize("fmt", FMTS)
def test_error_within_half_gap(fmt):
    S = F.FORMATS[fmt][0]
    mags = F.magnitudes(fmt).astype(np.float64)
    half_gap = np.diff(mags).max() / 2.0
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(64 * 64) * 0.02).astype(np.float32)
    codes, c = F.quantize(w, fmt)
    wh = oracle.bf16_bits_to_f32(F.dequant(codes, c, fmt)).astype(np.float64)
    cw = np.repeat(c.astype(np.float64), 64)
    bound = half_gap * cw / S * (1 + 2.0 ** -20) + np.abs(wh) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(w.astype(np.float64) - wh) <= bound)


def test_uniform_int4_mse_closed_form():
    # a fine uniform grid over [-c, c] in every block: MSE = (c / 7)^2 / 12 for a uniform step
    c = 0.7
    per = np.linspace(-c, c, 64, dtype=np.float64)
    rng = np.random.default_rng(3)
    blocks = []
    for _ in range(2000):
        b = per + rng.uniform(-c / 63, c / 63, 64)
        b[0], b[-1] = -c, c
        blocks.append(np.clip(b, -c, c))
    w = np.concatenate(blocks).astype(np.float32)
    codes, cc = F.quantize(w, "int4")
    st = F.error_stats(w, F.dequant(codes, cc, "int4"))
    assert abs(st["mse"] / ((c / 7) ** 2 / 12) - 1.0) < 0.03


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_block_and_sign_symmetry(fmt):
    w = np.zeros(128, dtype=np.float32)
    rng = np.random.default_rng(9)
    w[64:] = rng.standard_normal(64).astype(np.float32)
    codes, c = F.quantize(w, fmt)
    assert c[0] == 0 and np.all(codes[:64] == 0)
    assert np.all(F.dequant(codes, c, fmt)[:64] == 0)
    codes_n, c_n = F.quantize(-w, fmt)
    assert np.array_equal(c, c_n)
    nz = (codes & 7) != 0
    assert np.array_equal(codes_n[nz], codes[nz] ^ 8) and np.array_equal(codes_n[~nz], codes[~nz])
    a = oracle.bf16_bits_to_f32(F.dequant(codes, c, fmt))
    b = oracle.bf16_bits_to_f32(F.dequant(codes_n, c_n, fmt))
    assert np.array_equal(a, -b)


def test_bf16_rounding_matches_c_oracle():
    rng = np.random.default_rng(1)
    f = (rng.standard_normal(4000) * 10.0 ** rng.integers(-6, 6, 4000)).astype(np.float32)
    # exact ties between two bf16 values (low half 0x8000), both parities
    ties = (np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40A38000], dtype=np.uint32)).view(np.float32)
    f = np.concatenate([f, ties, np.float32([0.0, -0.0, 1.0, 65504.0])])
    assert np.array_equal(F.bf16_rne(f), oracle.f32_to_bf16_bits(f))


def nf4_stats(w):
    q = oracle.quantize(w)
    with_dq = F.error_stats(w, oracle.dequant(q))
    # the same codes with the exact fp32 absmax: the cost of double quantisation alone
    Q = oracle.codebook()
    codes = oracle.unpack_codes(q.codes, q.n)
    c1 = np.repeat(q.c1, 64)[: q.n]
    no_dq = F.error_stats(w, F.bf16_rne((Q[codes] * c1).astype(np.float32)))
    return with_dq, no_dq


def comparison(w):
    rows = {}
    rows["nf4_dq"], rows["nf4_exact_absmax"] = nf4_stats(w)
    for f in FMTS:
        codes, c = F.quantize(w, f)
        rows[f] = F.error_stats(w, F.dequant(codes, c, f))
    return rows


def test_format_comparison_gaussian(capsys):
    """Synthetic Gaussian weights (the pages' premise: weights are roughly normal), 2^18 values
    in 64-blocks, and the same with 0.1 % of the weights scaled by 10 (outliers)."""
    rng = np.random.default_rng(2024)
    w = (rng.standard_normal(1 << 18) * 0.02).astype(np.float32)
    wo = w.copy()
    idx = rng.choice(w.size, w.size // 1000, replace=False)
    wo[idx] *= 10.0
    out = {"gaussian": comparison(w), "gaussian_outliers": comparison(wo)}
    with capsys.disabled():
        for name, rows in out.items():
            print(f"\n{name}: format, normalised MSE, SNR dB, MSE / NF4+DQ MSE")
            base = rows["nf4_dq"]["mse"]
            for f, st in rows.items():
                print(f"  {f:18s} {st['nmse']:.5e} {st['snr_db']:7.3f} {st['mse'] / base:6.3f}")
    for rows in out.values():
        # NF4 + DQ beats the uniform Int4 grid on normal weights
        assert rows["nf4_dq"]["mse"] < rows["int4"]["mse"]
        # double quantisation of the constants costs little next to the 4-bit rounding itself
        # (0.03 % of the MSE on plain normal weights, about 2 % with outliers, whose absmax
        # constants spread wider and so get a coarser int8 step)
        assert rows["nf4_dq"]["mse"] < 1.05 * rows["nf4_exact_absmax"]["mse"]
