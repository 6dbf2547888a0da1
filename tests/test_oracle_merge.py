"""Pins of the oracle's adapter merge (page "QLoRA: put the large model in memory,
then change it with a small adapter", sections 5 and 6: merging the adapter into the
weight and re-quantising can change outputs). The merged BF16 weight is
w'[n,k] = bf16(fl(w^[n,k] + fl(s * d[n,k]))), d = the fused multiply-add chain of
A[k,j] * B[j,n] over j in increasing order, started from 0."""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def bf16_vals(x):
    return oracle.bf16_bits_to_f32(oracle.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))).reshape(np.shape(x))


def rn32(x: Fraction) -> np.float32:
    """x rounded to the nearest fp32, ties to the even significand (exact, via Fractions)."""
    c = np.float32(float(x))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - x),
                                     int(np.array(v, dtype=np.float32).view(np.uint32)) & 1))
    return np.float32(best)


def fmaf_exact(a, b, c):
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def problem(rows, cols, r, seed):
    g = np.random.default_rng(seed)
    w = oracle.f32_to_bf16_bits((g.standard_normal((rows, cols)) * 0.02).astype(np.float32)).reshape(rows, cols)
    A = bf16_vals(g.standard_normal((cols, r)) * 0.05)
    B = bf16_vals(g.standard_normal((r, rows)) * 0.05)
    return w, A, B


def test_merge_bruteforce_tiny():
    # every element against an exact emulation of the fused multiply-add chain
    w, A, B = problem(3, 5, 3, seed=1)
    s = np.float32(1.75)
    got = oracle.merge_bf16(w, A, B, float(s))
    wf = oracle.bf16_bits_to_f32(w).reshape(3, 5)
    for n in range(3):
        for k in range(5):
            d = np.float32(0.0)
            for j in range(3):
                d = fmaf_exact(A[k, j], B[j, n], d)
            t = np.float32(s * d)
            ref = oracle.f32_to_bf16_bits(np.array([np.float32(wf[n, k] + t)], dtype=np.float32))[0]
            assert got[n, k] == ref, (n, k)


def test_merge_rank_one_matches_fp32_arithmetic():
    # r = 1: d = fl(a*b) (+0), so the whole merge is plain fp32 arithmetic
    w, A, B = problem(64, 96, 1, seed=2)
    s = np.float32(2.0)
    got = oracle.merge_bf16(w, A, B, float(s))
    d = (A[:, 0][None, :] * B[0, :][:, None]).astype(np.float32) + np.float32(0.0)
    ref = oracle.f32_to_bf16_bits(oracle.bf16_bits_to_f32(w).reshape(w.shape) + (s * d).astype(np.float32))
    assert np.array_equal(got, ref.reshape(w.shape))


@pytest.mark.parametrize("which", ["s", "A"])
def test_merge_zero_adapter_is_identity(which):
    w, A, B = problem(32, 64, 8, seed=3)
    if which == "A":
        A = np.zeros_like(A)
    got = oracle.merge_bf16(w, A, B, 0.0 if which == "s" else 2.0)
    assert np.array_equal(got, w)


def test_merge_within_rounding_of_exact():
    # r = 64: the merged value is within the fp32 chain error and one bf16 rounding of
    # the exact w^ + s * (A B)^T
    w, A, B = problem(48, 80, 64, seed=4)
    s = 2.0
    got = oracle.bf16_bits_to_f32(oracle.merge_bf16(w, A, B, s)).reshape(w.shape).astype(np.float64)
    wf = oracle.bf16_bits_to_f32(w).reshape(w.shape).astype(np.float64)
    prod = (A.astype(np.float64) @ B.astype(np.float64)).T           # [rows, cols]
    absprod = (np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64))).T
    exact = wf + s * prod
    ulp_bf16 = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    bound = 0.5 * ulp_bf16 + s * 64 * 2.0 ** -24 * absprod + 2.0 ** -23 * np.abs(exact) + 1e-30
    assert np.all(np.abs(got - exact) <= 1.01 * bound)
