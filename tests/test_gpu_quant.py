"""GPU parity of quantisation, double quantisation and dequantisation against
the CPU oracle: codes, int8 constants, second-level constants, the offset and
the dequantised bf16 weights must match bit for bit."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def gpu_quantize(W):
    t = q.qlora_nf4_quantize(W)
    wh = q.qlora_nf4_dequant(t)
    st = q.qlora_get_device_status()
    return t, wh, st


def oracle_of(W):
    w32 = W.detach().float().cpu().numpy().reshape(W.shape[0], -1) if W.dim() == 2 else W.detach().float().cpu().numpy().reshape(1, -1)
    return oracle.quantize(w32)


def assert_bit_exact(W, t=None, wh=None):
    if t is None:
        t, wh, st = gpu_quantize(W)
        assert st == q.QLORA_OK
    ref = oracle_of(W)
    assert ref.status == 0
    assert np.array_equal(t.codes.cpu().numpy(), ref.codes), "codes"
    assert np.array_equal(t.scale8.cpu().numpy(), ref.scale8), "scale8"
    assert np.array_equal(t.scale2.cpu().numpy().view(np.uint32), ref.scale2.view(np.uint32)), "scale2"
    assert t.offset.cpu().numpy().view(np.uint32)[0] == np.float32(ref.offset).view(np.uint32), "offset"
    wh_ref = oracle.dequant(ref)
    got = wh.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    assert np.array_equal(got, wh_ref), "dequant"
    return ref


def test_tiny_layer_fp32():
    wl = si.workload("tiny")
    W = si.layer_inputs(wl, 0, device="cuda")["W"]
    assert_bit_exact(W)


@pytest.mark.parametrize("n", [1, 2, 3, 63, 64, 65, 127, 1000, 16384 + 37, 64 * 256, 64 * 256 + 64, 64 * 257 * 3 + 5])
def test_ragged_lengths(n):
    W = si.normal((1, n), 0.02, seed=n, device="cuda")
    assert_bit_exact(W)


@pytest.mark.parametrize("shape", [(7, 1000), (3, 5), (33, 4097)])
def test_ragged_shapes_bf16(shape):
    W = si.normal(shape, 0.02, seed=sum(shape), device="cuda", dtype=torch.bfloat16)
    assert_bit_exact(W)


def test_special_blocks():
    W = torch.zeros(4, 256, device="cuda")
    W[1, :64] = 0.5                  # constant positive block
    W[1, 64:128] = -0.25             # constant negative block
    W[2, 5] = -3.0                   # single nonzero block
    W[3, :] = torch.linspace(-1, 1, 256, device="cuda")
    assert_bit_exact(W)


def test_extreme_absmax_blocks():
    # blocks whose absmax has no normal reciprocal (subnormal, or above 2^125) take the
    # exact path; blocks just inside the range take the table; all match the oracle
    rng = np.random.default_rng(11)
    scales = [1e-45, 3e-40, 2.9e-39, 1.2e-38, 3e-38, 1e-30, 1.0, 4.2e37, 4.3e37, 1e38, 3.3e38]
    blocks = []
    for c in scales:
        b = (rng.standard_normal(64) * 0.3).astype(np.float32)
        b[rng.integers(64)] = 1.0
        blocks.append((b * np.float32(c)).astype(np.float32))
    w = np.concatenate(blocks)
    W = torch.from_numpy(w).view(1, -1).cuda()
    assert np.isfinite(w).all()
    assert_bit_exact(W)


def test_outliers_full_4096():
    wl = si.workload("l4096")
    W = si.layer_inputs(wl, 0, device="cuda", M=0)["W"]
    assert_bit_exact(W)


def test_midpoint_ties():
    # weights whose normalised value lands exactly on a decision threshold go
    # to the lower code on both sides
    T = oracle.midpoints()
    vals = np.concatenate([T, -T, [1.0, -1.0, 0.0]]).astype(np.float32)
    w = np.zeros(64 * 2, np.float32)
    w[: vals.size] = vals
    w[64: 64 + vals.size] = vals * np.float32(0.125)      # exact power-of-two rescale keeps the ties
    W = torch.from_numpy(w).view(1, -1).cuda()
    assert_bit_exact(W)


def test_nonfinite_sets_status():
    W = si.normal((4, 256), 0.02, seed=3, device="cuda")
    W[2, 17] = float("nan")
    t = q.qlora_nf4_quantize(W)
    assert q.qlora_get_device_status() == q.QLORA_ERR_NONFINITE
    assert q.qlora_get_device_status() == q.QLORA_OK       # read clears it
    W[2, 17] = float("inf")
    q.qlora_nf4_quantize(W, out=t)
    assert q.qlora_get_device_status() == q.QLORA_ERR_NONFINITE


def test_bounded_wait_reports_timeout():
    # a wait that nothing ends gives up after its limit, reports TIMEOUT through the
    # status word, and leaves the context usable (the next quantisation is exact)
    assert q.qlora_get_device_status() == q.QLORA_OK
    assert q.lib().qlora_selftest_wait_timeout(None) == q.QLORA_OK
    assert q.qlora_get_device_status() == q.QLORA_ERR_TIMEOUT
    assert q.qlora_get_device_status() == q.QLORA_OK       # read clears it
    W = si.normal((64, 256), 0.02, seed=9, device="cuda")
    t = q.qlora_nf4_quantize(W)
    assert q.qlora_get_device_status() == q.QLORA_OK
    ref = oracle.quantize(W.cpu().numpy())
    assert np.array_equal(t.codes.cpu().numpy(), ref.codes)


def test_reciprocal_approximation_within_one_ulp():
    # the fast code search is exact only while the hardware reciprocal stays within a few
    # ulps (its band is sized for 4); every mantissa of [1, 2) is measured
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert q.lib().qlora_selftest_rcp_error(out.data_ptr(), None) == q.QLORA_OK
    torch.cuda.synchronize()
    err_ulps = int(out.item()) / 1024.0
    assert err_ulps <= 1.0, err_ulps


def test_llama7b_layer_full_bf16():
    # every projection of one Llama-7B-shaped block, at full size
    wl = si.workload("llama7b", n_layers=1)
    for li in range(len(wl.layers)):
        W = si.layer_inputs(wl, li, device="cuda")["W"]
        assert_bit_exact(W)
        del W
        torch.cuda.empty_cache()


def test_largest_70b_projection_fp32():
    # the largest matrix of the 70B-like block (28672 x 8192, 235 M weights)
    wl = si.workload("l70b")
    li = [l.name for l in wl.layers].index("gate")
    W = si.layer_inputs(wl, li, device="cuda", M=0)["W"]
    assert_bit_exact(W)


def test_repeat_is_deterministic():
    W = si.normal((512, 1024), 0.02, seed=9, device="cuda")
    a = q.qlora_nf4_quantize(W)
    b = q.qlora_nf4_quantize(W)
    torch.cuda.synchronize()
    for x, y in [(a.codes, b.codes), (a.scale8, b.scale8), (a.scale2, b.scale2), (a.offset, b.offset)]:
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grouped_quantize_and_dequant(dtype):
    # a list of tensors through the grouped entry points: each tensor exactly as quantised
    # and dequantised alone (ragged sizes, a 1-weight tensor, a tensor of several groups)
    shapes = [(7, 1000), (1, 1), (512, 1024), (3, 5), (33, 4097), (64, 256 * 64 + 3), (1, 63)]
    Ws = [si.normal(sh, 0.02, seed=40 + i, device="cuda", dtype=dtype) for i, sh in enumerate(shapes)]
    ts = q.qlora_nf4_quantize_grouped(Ws)
    whs = q.qlora_nf4_dequant_grouped(ts)
    assert q.qlora_get_device_status() == q.QLORA_OK
    for W, t, wh in zip(Ws, ts, whs):
        assert_bit_exact(W, t, wh)


def test_grouped_more_than_one_launch_set():
    # more tensors than one launch takes (64): the list is cut into launch sets
    Ws = [si.normal((4, 64 * (1 + i % 5) + i), 0.02, seed=500 + i, device="cuda") for i in range(70)]
    ts = q.qlora_nf4_quantize_grouped(Ws)
    whs = q.qlora_nf4_dequant_grouped(ts)
    assert q.qlora_get_device_status() == q.QLORA_OK
    for W, t, wh in zip(Ws, ts, whs):
        assert_bit_exact(W, t, wh)


def _band_weights_fp32(rng):
    # blocks [c1, w_1 .. w_63]: w = fl(T[t] c1) moved by k fp32 ulps (k = -6 .. 6), with c1
    # not a power of two, so the normalised weight lands within a few ulps of a threshold
    T = oracle.midpoints().astype(np.float32)
    blocks = []
    for c1 in np.float32([0.7, 0.3, 1.3, 2.7, 0.05, 123.4, 0.0171, 9.9e-4]) * np.float32(1 + rng.random(8) * 1e-3):
        vals = []
        for thr in T:
            base = np.float32(thr * c1)
            for k in range(-6, 7):
                w = base
                step = np.float32(np.inf if k > 0 else -np.inf)
                for _ in range(abs(k)):
                    w = np.nextafter(w, step, dtype=np.float32)
                if abs(w) <= c1:
                    vals.append(w)
        vals = np.array(vals, np.float32)
        for j in range(0, vals.size, 63):
            blk = np.zeros(64, np.float32)
            blk[0] = c1
            part = vals[j: j + 63]
            blk[1: 1 + part.size] = part
            blocks.append(blk)
    return np.concatenate(blocks)


def _band_weights_bf16():
    # bf16 pairs (c1, w), searched over every bf16 mantissa of c1, whose fp32 quotient lies
    # nearest to a threshold. With 8-bit operands no quotient comes within 16 fp32 ulps of a
    # threshold (the search shows it), so bf16 input never reaches the 4-ulp fallback band;
    # the pairs within 256 ulps are the closest there are. Blocks [c1 2^e, w 2^e, 0 ...].
    T = oracle.midpoints().astype(np.float32)
    c1 = torch.arange(0x3f80, 0x4000, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float().numpy()
    hits, closest = [], np.inf
    for thr in T:
        approx = torch.from_numpy((thr * c1).astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
        for d in range(-3, 4):
            w = torch.from_numpy((approx.astype(np.int32) + d).astype(np.int16)).view(torch.bfloat16).float().numpy()
            x = (w / c1).astype(np.float32)          # IEEE single division, correctly rounded
            dist = np.abs(x - thr) / np.spacing(np.abs(thr)).astype(np.float32)
            ok = (dist <= 256) & (np.abs(w) <= c1)
            closest = min(closest, float(dist[np.abs(w) <= c1].min()))
            hits.extend(zip(c1[ok], w[ok]))
    blocks = []
    for e in (-6, -2, 0, 3):
        for c, w in hits:
            blk = np.zeros(64, np.float32)
            blk[0], blk[1] = np.ldexp(c, e), np.ldexp(w, e)
            blocks.append(blk)
    return np.concatenate(blocks), len(hits), closest


@pytest.mark.parametrize("divide_every_weight", [0, 1])
def test_threshold_band_both_code_searches(divide_every_weight):
    # weights whose normalised value lies within a few ulps of a decision threshold: the
    # bin table's u (about w / c1 / 2 + 1/2, from an approximate 1/c1) is then inside its
    # fallback band (within 2^-22 of fl(T/2 + 1/2), about 2^-21 of T), where the exact
    # quotient decides. Both code searches (table with fallback; a division per weight)
    # must match the oracle bit for bit, in fp32 and for the closest bf16 pairs.
    rng = np.random.default_rng(5)
    w32 = _band_weights_fp32(rng)
    wb, nhits, closest = _band_weights_bf16()
    assert nhits >= 10 and closest > 16
    # the fp32 set really reaches the band: w times fl(1/c1) within |T| 2^-21 of T (inside
    # the band, since |T| < 1) for many of its weights
    c1 = np.repeat(w32.reshape(-1, 64)[:, 0], 64)
    xa = (w32 * (np.float32(1) / c1)).astype(np.float32)
    T = oracle.midpoints().astype(np.float32)
    near = np.min(np.abs(xa[:, None] - T[None, :]) - np.abs(T)[None, :] * np.float32(2.0 ** -21), axis=1) <= 0
    assert near.sum() > 500
    q.lib().qlora_nf4_set_code_search(divide_every_weight)
    try:
        assert_bit_exact(torch.from_numpy(w32).view(1, -1).cuda())
        assert_bit_exact(torch.from_numpy(wb).view(1, -1).cuda().to(torch.bfloat16))
    finally:
        q.lib().qlora_nf4_set_code_search(0)
