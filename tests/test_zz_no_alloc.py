"""The quantiser entry point that allocates nothing (qlora_nf4_quantize_noalloc).

It exists for callers that cannot allocate device memory and so cannot pass the
workspace qlora_nf4_quantize needs; its scratch is a fixed array inside the
library. Called here straight through the C ABI (ctypes), twice in a row on
different weights, and compared with the workspace entry point: the format is
an exact encoding, so the two must agree bit for bit (the tolerance the other
quantiser tests use). This file is collected last on purpose."""
import ctypes

import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import synth_inputs as si

pytestmark = pytest.mark.gpu


def _noalloc(W, dt):
    rows, cols = W.shape
    out = q.nf4_empty(rows, cols, W.device)
    t = out.ctype()
    st = q.lib().qlora_nf4_quantize_noalloc(ctypes.c_void_p(W.data_ptr()), dt, ctypes.byref(t),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _same(a, b):
    torch.cuda.synchronize()
    return all(torch.equal(x, y) for x, y in ((a.codes, b.codes), (a.scale8, b.scale8),
                                                (a.scale2, b.scale2), (a.offset, b.offset)))


def test_noalloc_matches_workspace_entry_two_calls():
    # a large fp32 matrix first, then a smaller ragged bf16 one: the second call
    # must not be affected by what the first left in the shared scratch
    W1 = si.normal((4096, 4096), 0.02, seed=11, device="cuda")
    W2 = si.normal((33, 4097), 0.02, seed=12, device="cuda", dtype=torch.bfloat16)
    for W, dt in ((W1, q.QLORA_F32), (W2, q.QLORA_BF16)):
        st, got = _noalloc(W, dt)
        assert st == q.QLORA_OK
        ref = q.qlora_nf4_quantize(W)
        assert q.qlora_get_device_status() == q.QLORA_OK
        assert _same(got, ref)


def test_noalloc_rejects_tensors_above_limit():
    # 2^26 + 64 weights: rejected on the host before any launch
    fake = 1 << 20
    t = q._Tensor(1, (1 << 26) + 64, fake, fake, fake, fake)
    st = q.lib().qlora_nf4_quantize_noalloc(ctypes.c_void_p(fake), q.QLORA_F32, ctypes.byref(t), None)
    assert st == q.QLORA_ERR_UNSUPPORTED_SHAPE
