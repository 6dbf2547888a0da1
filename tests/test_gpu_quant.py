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
