"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test states what fixes the expected value: a number printed on the pages
(fixtures under tests/golden, each with its citation), a closed form, an
invariant of the definition, a library routine, or brute force on small inputs.
Source page: "QLoRA: put the large model in memory, then change it with a small
adapter" (wq-win.github.io/llm/074-qlora), sections 1-3.
"""
import math

import numpy as np
import pytest
import torch
from scipy.stats import norm

import oracle

DELTA = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


# ---------------------------------------------------------------- codebook
def test_quantile_solver_matches_library():
    # the bisection quantile against scipy's normal quantile (a library routine)
    for p in [0.5, 0.51, 0.6, 0.75, 0.9, DELTA, 0.99, 0.999]:
        assert abs(oracle.norm_quantile_upper(p) - norm.ppf(p)) < 1e-12


def test_codebook_structure():
    # section 2: sixteen values, exact zero, normalised by absmax to [-1, 1],
    # finer spacing near zero than in the tails
    Q = oracle.codebook()
    assert Q.shape == (16,) and Q.dtype == np.float32
    assert np.all(np.diff(Q) > 0), "strictly increasing"
    assert Q[7].view(np.uint32) == 0, "exact +0.0 at code 7"
    assert Q[0] == -1.0 and Q[15] == 1.0
    gaps = np.diff(Q.astype(np.float64))
    # positive side: gaps grow from zero outwards; negative side likewise
    assert np.all(np.diff(gaps[7:]) > 0)
    assert np.all(np.diff(gaps[:7][::-1]) > 0)
    # 8 positive values, 7 negative values
    assert np.sum(Q > 0) == 8 and np.sum(Q < 0) == 7


def test_codebook_quantile_property():
    # every entry is a normal quantile at equally spaced probabilities
    # (8 steps on the positive side, 7 on the negative side, ending at delta),
    # checked through scipy's normal CDF
    Qd = oracle.codebook_f64()
    z = norm.ppf(DELTA)
    pos = norm.cdf(Qd[7:] * z)            # codes 7..15
    neg = norm.cdf(-Qd[:8][::-1] * z)     # codes 7..0, mirrored
    assert np.allclose(np.diff(pos), (DELTA - 0.5) / 8, rtol=0, atol=1e-12)
    assert np.allclose(np.diff(neg), (DELTA - 0.5) / 7, rtol=0, atol=1e-12)
    assert abs(pos[0] - 0.5) < 1e-15 and abs(pos[-1] - DELTA) < 1e-12


def test_codebook_fp32_rounding_unambiguous():
    # the fp32 table is the single rounding of the double values, and no value is
    # close enough to an fp32 rounding boundary for a 1e-12 error to flip it
    Qd = oracle.codebook_f64()
    Q = oracle.codebook()
    assert np.array_equal(Qd.astype(np.float32), Q)
    for d, f in zip(Qd, Q):
        if d == 0.0 or abs(d) == 1.0:
            continue
        up = np.nextafter(f, np.float32(np.inf))
        dn = np.nextafter(f, np.float32(-np.inf))
        lo_b = (float(f) + float(dn)) / 2
        hi_b = (float(f) + float(up)) / 2
        margin = min(abs(d - lo_b), abs(hi_b - d)) / abs(d)
        assert margin > 1e-12


# ---------------------------------------------------------------- byte counts
def test_worked_example_16384(golden):
    g = golden("worked_example_16384.txt")
    n = g["n_weights"]
    w = np.random.default_rng(1).standard_normal(n).astype(np.float32) * 0.02
    q = oracle.quantize(w, 1, n)
    assert q.scale8.size == g["blocks_of_64"]
    assert q.codes.nbytes == g["code_bytes"]
    assert q.c1.nbytes == g["fp32_constant_bytes"]
    assert q.scale8.nbytes == g["int8_constant_bytes"]
    assert q.scale2.nbytes == g["second_level_constant_bytes"]
    dq = q.scale8.nbytes + q.scale2.nbytes
    assert dq == g["double_quant_constant_bytes"]
    assert q.c1.nbytes - dq == g["bytes_saved"]
    # the stored format adds the 4-byte offset
    assert oracle.storage_bytes(1, n) == g["code_bytes"] + dq + 4


def test_cost_model_bits(golden):
    g = golden("cost_model_bits.txt")
    exact = 8 / 64 + 32 / (64 * 256)
    assert abs(exact - g["double_quant_bits_approx"]) < g["approx_tolerance"]
    assert abs((g["single_level_bits"] - exact) - g["saving_bits_approx"]) < g["approx_tolerance"]
    # the format's own byte count reproduces the model exactly when n is a
    # multiple of 64*256 (offset excluded, as the page excludes it)
    for rows, cols in [(4096, 4096), (11008, 4096), (4096, 11008), (1024, 8192), (28672, 8192)]:
        n = rows * cols
        bits = (oracle.storage_bytes(rows, cols) - 4) * 8 / n
        assert bits == 4 + exact
        assert abs(bits - g["total_bits_approx"]) < g["approx_tolerance"]


def test_lora_count(golden):
    g = golden("lora_4096_r64.txt")
    assert g["d_in"] * g["d_out"] == g["base_params"]
    assert g["base_params"] * 2 == g["base_bytes_16bit"]
    assert oracle.sizes(g["d_out"], g["d_in"])[1] == g["base_code_bytes_4bit"]
    cnt = oracle.lora_param_count(g["d_in"], g["d_out"], g["rank"])
    assert cnt == g["lora_params"]
    assert 100.0 * cnt / g["base_params"] == g["lora_percent"]


# ---------------------------------------------------------------- code search
def test_nearest_code_bruteforce_random():
    rng = np.random.default_rng(7)
    rows, cols = 8, 192
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    q = oracle.quantize(w)
    codes = oracle.unpack_codes(q.codes, w.size)
    Q = oracle.codebook().astype(np.float64)
    T = oracle.midpoints()
    flat = w.ravel()
    for i in range(flat.size):
        c1 = q.c1[i // 64]
        x = np.float32(flat[i]) / np.float32(c1)     # IEEE fp32 division
        d = np.abs(float(x) - Q)
        best = int(np.argmin(d))                      # ties resolve to the lower index
        if codes[i] != best:
            assert np.any(T == x), (i, float(x), codes[i], best)
            assert codes[i] == best - 1


@pytest.mark.slow
def test_exhaustive_fp32_sweep():
    bad, tested, onthr = oracle.sweep_codes()
    assert tested == 2 * (0x3F800000 + 1)
    assert bad == 0
    assert onthr <= 15


def test_threshold_tie_goes_low_and_negative_zero():
    Q = oracle.codebook()
    T = oracle.midpoints(Q)
    for t in range(15):
        assert oracle.code_of(float(T[t]), T) == t
        assert oracle.code_of(float(np.nextafter(T[t], np.float32(2))), T) == t + 1
    assert oracle.code_of(-0.0, T) == 7
    assert oracle.code_of(0.0, T) == 7


# ---------------------------------------------------------------- blocks
def test_special_blocks():
    # zero block: absmax 0, every code is the zero code, dequantised to zero
    q = oracle.quantize(np.zeros(128, np.float32), 1, 128)
    assert np.all(q.codes == 0x77) and np.all(q.c1 == 0)
    assert np.all(oracle.bf16_bits_to_f32(oracle.dequant(q)) == 0)
    # constant positive / negative block: every element is the absmax
    q = oracle.quantize(np.full(64, 0.5, np.float32), 1, 64)
    assert np.all(oracle.unpack_codes(q.codes, 64) == 15)
    q = oracle.quantize(np.full(64, -0.5, np.float32), 1, 64)
    assert np.all(oracle.unpack_codes(q.codes, 64) == 0)
    # one nonzero element
    w = np.zeros(64, np.float32)
    w[5] = -3.0
    q = oracle.quantize(w, 1, 64)
    c = oracle.unpack_codes(q.codes, 64)
    assert c[5] == 0 and np.all(np.delete(c, 5) == 7)
    assert q.c1[0] == 3.0


def test_absmax_element_roundtrip():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(64 * 300) * 0.02).astype(np.float32)
    q = oracle.quantize(w, 1, w.size)
    codes = oracle.unpack_codes(q.codes, w.size)
    wh = oracle.bf16_bits_to_f32(oracle.dequant(q))
    ch = oracle.dequant_constants(q)
    for b in range(q.c1.size):
        blk = w[64 * b: 64 * b + 64]
        i = int(np.argmax(np.abs(blk)))
        assert abs(blk[i]) == q.c1[b]
        want_code = 15 if blk[i] > 0 else 0
        assert codes[64 * b + i] == want_code
        assert wh[64 * b + i] == oracle.bf16_bits_to_f32(
            np.array([oracle.f32_to_bf16_bits(np.float32(np.sign(blk[i])) * ch[b])[0]]))[0]


def test_ragged_sizes_and_padding():
    rng = np.random.default_rng(3)
    n = 16384 + 37
    w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    q = oracle.quantize(w, 1, n)
    assert q.codes.size == (n + 1) // 2
    assert q.scale8.size == 257 and q.scale2.size == 2
    assert q.codes[-1] & 15 == 7            # odd n: pad nibble is the zero code
    assert q.c1[-1] == np.max(np.abs(w[256 * 64:]))
    # dequant of the ragged tensor equals dequant of the same data padded with zeros
    # in all positions that exist
    wh = oracle.dequant(q)
    assert wh.size == n


# ---------------------------------------------------------------- offset
def test_offset_is_mean_of_constants():
    rng = np.random.default_rng(5)
    for nb in [1, 2, 255, 256, 257, 1000, 4099]:
        c1 = (np.abs(rng.standard_normal(nb)) * 0.05).astype(np.float32)
        mu = oracle.offset(c1)
        exact = math.fsum(float(v) for v in c1) / nb        # correctly rounded sum
        f = np.float32(exact)
        assert abs(float(mu) - exact) <= abs(float(np.nextafter(f, np.float32(np.inf))) - float(f))


def test_pairwise_tree_order():
    # hand-derived sums that separate the pairwise tree from left-to-right summation
    big = 2.0 ** 53
    # tree: (big + 1) + (1 + 1) = big + 2 ; sequential: ((big+1)+1)+1 = big
    assert oracle.pairwise_sum_f64(np.array([big, 1, 1, 1])) == big + 2
    # odd length: ((big+1) + (1+1)) + (1 + 0) = (big+2)+1 -> rounds to big+4 (ties to even)
    assert oracle.pairwise_sum_f64(np.array([big, 1, 1, 1, 1])) == big + 4
    assert oracle.pairwise_sum_f64(np.array([1.0, 2.0, 3.0])) == 6.0
    assert oracle.pairwise_sum_f64(np.array([7.5])) == 7.5


# ---------------------------------------------------------------- double quant
def test_double_quant_bounds():
    rng = np.random.default_rng(9)
    rows, cols = 64, 1024
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    w[rng.random((rows, cols)) < 0.001] *= 10
    q = oracle.quantize(w)
    assert q.scale8.min() >= -127 and q.scale8.max() <= 127
    ch = oracle.dequant_constants(q)
    for b in range(q.c1.size):
        s2 = float(q.scale2[b // 256])
        ulp = np.spacing(np.float32(max(abs(q.c1[b]), abs(q.offset), abs(ch[b]))))
        assert abs(float(ch[b]) - float(q.c1[b])) <= s2 / 254 * (1 + 1e-5) + 4 * float(ulp)
    # each second-level group uses the full int8 range on its largest deviation
    for j in range(q.scale2.size):
        grp = q.scale8[256 * j: 256 * j + 256]
        if q.scale2[j] > 0:
            assert np.max(np.abs(grp.astype(int))) == 127


def test_weight_error_bound():
    rng = np.random.default_rng(13)
    w = (rng.standard_normal(64 * 512) * 0.02).astype(np.float32)
    q = oracle.quantize(w, 1, w.size)
    wh = oracle.bf16_bits_to_f32(oracle.dequant(q)).astype(np.float64)
    ch = oracle.dequant_constants(q).astype(np.float64)
    gmax = float(np.max(np.diff(oracle.codebook().astype(np.float64))))
    for b in range(q.c1.size):
        c1 = float(q.c1[b])
        blk = slice(64 * b, 64 * b + 64)
        err = np.abs(wh[blk] - w[blk].astype(np.float64))
        bound = c1 * gmax / 2 + abs(ch[b] - c1) + np.abs(wh[blk]) * 2.0 ** -8 + 1e-7 * c1
        assert np.all(err <= bound)


def test_bf16_rounding_matches_library():
    # round-to-nearest-even to bf16 against torch's conversion (a library routine),
    # including exact ties
    rng = np.random.default_rng(17)
    f = (rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000)).astype(np.float32)
    ties = (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    f = np.concatenate([f, ties, -ties, np.float32([0.0, -0.0, 1e-45, 3.4e38])])
    ours = oracle.f32_to_bf16_bits(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------- products
def _tiny_problem(seed=0, M=3, d_in=64, d_out=16, r=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, d_in))
    Ws = rng.standard_normal((d_out, d_in)) * 0.1
    A = rng.standard_normal((d_in, r)) * 0.1
    B = rng.standard_normal((r, d_out)) * 0.1
    dY = rng.standard_normal((M, d_out))
    return X, Ws, A, B, dY


def test_backward_matches_finite_differences():
    # section 1: dX flows through W^ transposed; A and B get gradients; the base does not
    X, Ws, A, B, dY = _tiny_problem()
    s = 1.7

    def loss(X_, A_, B_):
        return float(np.sum(oracle.linear_fwd(X_, Ws, A_, B_, s) * dY))

    dX, dA, dB = oracle.linear_bwd(X, dY, Ws, A, B, s)
    h = 1e-6
    for arr, grad, name in [(X, dX, "X"), (A, dA, "A"), (B, dB, "B")]:
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = loss(X, A, B)
            arr[idx] = old - h
            lm = loss(X, A, B)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - grad)) <= 1e-6 * max(1.0, np.max(np.abs(grad))), name


def test_forward_reduces_to_plain_matmul():
    X, Ws, A, B, dY = _tiny_problem(1)
    ref = torch.matmul(torch.from_numpy(X), torch.from_numpy(Ws).T).numpy()
    assert np.allclose(oracle.linear_fwd(X, Ws, A, B, 0.0), ref, rtol=1e-14, atol=1e-14)
    assert np.allclose(oracle.linear_fwd(X, Ws, A, np.zeros_like(B), 2.0), ref, rtol=1e-14, atol=1e-14)


def test_dx_base_term_is_transposed_forward():
    X, Ws, A, B, dY = _tiny_problem(2)
    dX, _, _ = oracle.linear_bwd(X, dY, Ws, A, B, 0.0)
    r = A.shape[1]
    zA, zB = np.zeros((Ws.shape[0], r)), np.zeros((r, Ws.shape[1]))
    assert np.allclose(dX, oracle.linear_fwd(dY, Ws.T, zA, zB, 0.0), rtol=1e-14, atol=1e-14)
