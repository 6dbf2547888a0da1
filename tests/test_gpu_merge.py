"""GPU parity of the adapter merge and re-quantisation (page "QLoRA: put the large
model in memory, then change it with a small adapter", sections 5 and 6): the merged
BF16 weight and its NF4 + double quantisation must match the oracle bit for bit, and
the change of the layer's output is measured."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_merge(W, A, B, s, in_place=False):
    t = q.qlora_nf4_quantize(W)
    ref = oracle.quantize(W.float().cpu().numpy())
    rows, cols = W.shape
    w_hat = oracle.dequant(ref).reshape(rows, cols)
    An = A.float().cpu().numpy()
    Bn = B.float().cpu().numpy()
    merged_ref = oracle.merge_bf16(w_hat, An, Bn, s)
    out, wb = q.qlora_nf4_merge_adapter(t, A, B, s, out=t if in_place else None)
    assert q.qlora_get_device_status() == q.QLORA_OK
    assert np.array_equal(bits(wb), merged_ref), "merged bf16"
    rq = oracle.quantize_bf16(merged_ref.ravel(), rows, cols)
    assert np.array_equal(out.codes.cpu().numpy(), rq.codes), "codes"
    assert np.array_equal(out.scale8.cpu().numpy(), rq.scale8), "scale8"
    assert np.array_equal(out.scale2.cpu().numpy().view(np.uint32), rq.scale2.view(np.uint32)), "scale2"
    assert out.offset.cpu().numpy().view(np.uint32)[0] == np.float32(rq.offset).view(np.uint32), "offset"
    return out


@pytest.mark.parametrize("rows,cols,r", [(100, 192, 8), (64, 64, 1), (257, 320, 24), (128, 256, 256),
                                         (300, 448, 40), (1, 64, 33)])
def test_merge_small_ragged(rows, cols, r):
    W = si.normal((rows, cols), 0.02, seed=rows + cols, device="cuda")
    A = si.normal((cols, r), 0.05, seed=rows + 1, device="cuda", dtype=torch.bfloat16)
    B = si.normal((r, rows), 0.05, seed=rows + 2, device="cuda", dtype=torch.bfloat16)
    check_merge(W, A, B, 2.0)


def test_merge_in_place():
    W = si.normal((192, 256), 0.02, seed=5, device="cuda")
    A = si.normal((256, 16), 0.05, seed=6, device="cuda", dtype=torch.bfloat16)
    B = si.normal((16, 192), 0.05, seed=7, device="cuda", dtype=torch.bfloat16)
    check_merge(W, A, B, 1.5, in_place=True)


def test_merge_4096_layer_and_output_change():
    # the bench's 4096 x 4096 layer with its rank-64 adapter; the merged-and-requantised
    # weight changes the output by the re-quantisation error of the adapter term
    wl = si.workload("l4096")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0, device="cuda")
    out = check_merge(inp["W"], inp["A"], inp["B"], L.s)
    t = q.qlora_nf4_quantize(inp["W"])
    X = inp["X"][:256]
    Y_unmerged, _ = q.qlora_linear_fwd(X, t, inp["A"], inp["B"], L.s)
    Y_merged, _ = q.qlora_linear_fwd(X, out, None, None, 0.0)
    ref = Y_unmerged.double()
    diff = (Y_merged.double() - ref)
    rel_fro = (diff.norm() / ref.norm()).item()
    assert np.isfinite(rel_fro) and rel_fro < 0.5
