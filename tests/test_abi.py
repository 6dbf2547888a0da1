"""The C-ABI library loads, exports every declared entry point, and its
host-side logic (sizes, workspace queries, argument checks, the codebook
derivation) behaves as declared. No GPU compute is called here."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_nf4_quantized_double_b200 as q
import oracle

DEFAULT_PAIR_MIN_M = 128   # the library's default token count for the pair-GEMM route

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(qlora_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = q.lib()
    names = declared_functions()
    assert len(names) >= 11
    for name in names:
        assert hasattr(L, name), name
    # the binding wraps every declared function
    for name in names:
        assert name in q._SIGS, name


def test_codebook_bit_equal_to_oracle():
    # the library derives its codebook on the host (Newton on erfc), the
    # oracle by bisection; the fp32 tables must agree bit for bit
    lib_q = np.array(q.qlora_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(lib_q.view(np.uint32), oracle.codebook().view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(1, 1), (1, 16384), (512, 256), (4096, 4096), (11008, 4096),
                                       (3, 16421), (28672, 8192)])
def test_storage_bytes_match_format(rows, cols):
    assert q.qlora_nf4_storage_bytes(rows, cols) == oracle.storage_bytes(rows, cols)


def test_storage_bytes_invalid():
    assert q.qlora_nf4_storage_bytes(0, 5) == 0
    assert q.qlora_nf4_storage_bytes(5, -1) == 0


def test_quantize_workspace_size():
    L = q.lib()
    n, _, nb, nb2 = q.nf4_sizes(4096, 4096)
    ws = L.qlora_nf4_quantize_workspace(4096, 4096)
    assert ws >= nb * 4 + nb2 * 8
    assert L.qlora_nf4_quantize_workspace(0, 1) == 0


def test_workspace_queries_positive():
    L = q.lib()
    for M in (1, 16, 17, 4096):
        assert L.qlora_linear_fwd_workspace(M, 4096, 4096, 64) > 0
        assert L.qlora_linear_bwd_workspace(M, 4096, 4096, 64) > 0
    # from 128 tokens on the pair GEMM runs: the bf16 weight in the workspace, here 64 whole
    # 256 x 256 tiles (no split)
    assert L.qlora_linear_bwd_workspace(256, 4096, 16384, 0) == 4096 * 16384 * 2
    # ... and a dgrad with only 16 tiles splits each tile's K blocks 4 ways: the bf16 weight
    # plus fp32 partials (148 SMs, the count assumed without a GPU)
    assert L.qlora_linear_bwd_workspace(256, 4096, 4096, 0) == 4096 * 4096 * 2 + 4 * 256 * 4096 * 4
    # under 128 tokens the fused kernels always run; from 128 on the pair route (forward too)
    assert L.qlora_linear_bwd_workspace(127, 4096, 4096, 0) == 0
    assert L.qlora_linear_fwd_workspace(127, 11008, 4096, 0) == 0
    assert L.qlora_linear_fwd_workspace(128, 11008, 4096, 0) >= 11008 * 4096 * 2
    assert L.qlora_linear_bwd_workspace(128, 4096, 11008, 0) >= 4096 * 11008 * 2
    # with P raised to 512, a batch of 256 whose fused kernel fills the SMs stages nothing
    L.qlora_linear_set_pair_min_m(512)
    try:
        assert L.qlora_linear_bwd_workspace(256, 4096, 16384, 0) == 0
        assert L.qlora_linear_bwd_workspace(256, 4096, 4096, 0) == 4096 * 4096 * 2 + 4 * 256 * 4096 * 4
    finally:
        L.qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)
    # at 4096 tokens the layer keeps a bf16 copy of the dequantised weight
    assert L.qlora_linear_bwd_workspace(4096, 4096, 4096, 0) == 4096 * 4096 * 2
    assert L.qlora_linear_fwd_workspace(4096, 4096, 4096, 0) == 4096 * 4096 * 2


def test_grouped_forward_host_checks():
    # argument checks of the grouped entry point run on the host (no GPU needed)
    L = q.lib()
    fake = 1 << 20
    t = q._Tensor(64, 64, fake, fake, fake, fake)
    d = (q._LinearDesc * 2)(q._LinearDesc(fake, ctypes.pointer(t), None, None, 0, 1.0, fake, None),
                            q._LinearDesc(fake, ctypes.pointer(t), None, None, 0, 1.0, fake, None))
    assert L.qlora_linear_fwd_grouped(1, 0, d, None, 0, None) == q.QLORA_ERR_INVALID_ARG
    # two 64 x 64 items at M = 1: one K chunk each, so fp32 sums [1][64][1] per item, each
    # region 256-byte aligned
    assert L.qlora_linear_fwd_grouped_workspace(1, 2, d) == 2 * 256
    # 64 x 4096 (two K chunks of 2048) at M = 3 with rank 8: the fp32 chunk sums [2][64][3]
    # and the X A partials of 32 128-input chunks [32][3][8], each region 256-byte aligned
    t2 = q._Tensor(64, 4096, fake, fake, fake, fake)
    d2 = (q._LinearDesc * 1)(q._LinearDesc(fake, ctypes.pointer(t2), fake, fake, 8, 1.0, fake, None))
    assert L.qlora_linear_fwd_grouped_workspace(3, 1, d2) == 2 * 64 * 3 * 4 + 32 * 3 * 8 * 4
    assert L.qlora_linear_fwd_grouped(1, 2, d, None, 0, None) == q.QLORA_ERR_WORKSPACE
    bad = (q._LinearDesc * 1)(q._LinearDesc(fake, ctypes.pointer(q._Tensor(64, 100, fake, fake, fake, fake)),
                                            None, None, 0, 1.0, fake, None))
    assert L.qlora_linear_fwd_grouped(1, 1, bad, None, 0, None) == q.QLORA_ERR_UNSUPPORTED_SHAPE


def test_status_strings():
    for s in range(7):
        assert len(q.status_string(s)) > 0
    assert q.status_string(99) == "unknown status"


def test_argument_checks_run_on_host():
    # null and misaligned pointers, bad shapes and a missing workspace are
    # rejected before any launch, so these calls need no GPU
    L = q.lib()
    t = q._Tensor(64, 64, 0, 0, 0, 0)
    assert L.qlora_nf4_quantize(None, 0, ctypes.byref(t), None, 0, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_dequant(ctypes.byref(t), None, None) == q.QLORA_ERR_INVALID_ARG
    fake = 1 << 20   # never dereferenced: validation fails first
    good = q._Tensor(64, 64, fake, fake, fake, fake)
    assert L.qlora_nf4_quantize(ctypes.c_void_p(fake), 7, ctypes.byref(good), None, 0, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(ctypes.c_void_p(fake + 4), 0, ctypes.byref(good), None, 0, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_nf4_quantize(ctypes.c_void_p(fake), 0, ctypes.byref(good), None, 0, None) == q.QLORA_ERR_WORKSPACE
    bad_cols = q._Tensor(64, 100, fake, fake, fake, fake)
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(bad_cols), None, None, 0, 1.0,
                              ctypes.c_void_p(fake), None, None, 0, None) == q.QLORA_ERR_UNSUPPORTED_SHAPE
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(good), ctypes.c_void_p(fake),
                              ctypes.c_void_p(fake), 12, 1.0, ctypes.c_void_p(fake), None, None, 0,
                              None) == q.QLORA_ERR_UNSUPPORTED_SHAPE          # r % 8 != 0
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(good), ctypes.c_void_p(fake),
                              ctypes.c_void_p(fake), 16, float("nan"), ctypes.c_void_p(fake), None, None, 0,
                              None) == q.QLORA_ERR_INVALID_ARG                # non-finite scale
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(good), ctypes.c_void_p(fake),
                              ctypes.c_void_p(fake), 16, 1.0, ctypes.c_void_p(fake), None, None, 0,
                              None) == q.QLORA_ERR_WORKSPACE
    assert L.qlora_linear_bwd(None, ctypes.c_void_p(fake), 0, ctypes.byref(good), None, None, 0, 1.0, None,
                              ctypes.c_void_p(fake), None, None, None, 0, None) == q.QLORA_ERR_UNSUPPORTED_SHAPE
    # an empty batch, a row count that is not a multiple of 16, a rank above 256
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 0, ctypes.byref(good), None, None, 0, 1.0,
                              ctypes.c_void_p(fake), None, None, 0, None) == q.QLORA_ERR_UNSUPPORTED_SHAPE
    bad_rows = q._Tensor(40, 64, fake, fake, fake, fake)
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(bad_rows), None, None, 0, 1.0,
                              ctypes.c_void_p(fake), None, None, 0, None) == q.QLORA_ERR_UNSUPPORTED_SHAPE
    assert L.qlora_linear_fwd(ctypes.c_void_p(fake), 4, ctypes.byref(good), ctypes.c_void_p(fake),
                              ctypes.c_void_p(fake), 264, 1.0, ctypes.c_void_p(fake), None, None, 0,
                              None) == q.QLORA_ERR_UNSUPPORTED_SHAPE


def test_fmt4_argument_checks_run_on_host():
    L = q.lib()
    fake = ctypes.c_void_p(1 << 20)
    assert L.qlora_fmt4_quantize(None, 0, 64, 0, fake, fake, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_fmt4_quantize(fake, 0, 0, 0, fake, fake, None) == q.QLORA_ERR_INVALID_ARG       # n < 1
    assert L.qlora_fmt4_quantize(fake, 0, 64, 5, fake, fake, None) == q.QLORA_ERR_INVALID_ARG      # format
    assert L.qlora_fmt4_quantize(fake, 2, 64, 0, fake, fake, None) == q.QLORA_ERR_INVALID_ARG      # dtype
    assert L.qlora_fmt4_quantize(ctypes.c_void_p((1 << 20) + 2), 0, 64, 0, fake, fake, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_fmt4_dequant(fake, fake, 64, 1, ctypes.c_void_p((1 << 20) + 2), None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_fmt4_dequant(ctypes.c_void_p((1 << 20) + 8), fake, 64, 1, fake, None) == q.QLORA_ERR_INVALID_ARG


def test_grouped_workspace_is_largest_group_of_eight():
    # more than eight projections go in groups of eight that reuse one workspace, so the
    # query returns the largest group's need, and a group of one equals the single call's
    L = q.lib()
    fake = 1 << 20
    shapes = [(4096, 4096, 16)] * 4 + [(11008, 4096, 0)] * 2 + [(4096, 11008, 0)] + [(1024, 2048, 64)] * 13
    ts = [q._Tensor(rows, cols, fake, fake, fake, fake) for rows, cols, _ in shapes]
    descs = [q._LinearDesc(fake, ctypes.pointer(t), fake, fake, r, 1.0, fake, None) for t, (_, _, r) in zip(ts, shapes)]
    for M in (1, 16):
        arr = (q._LinearDesc * len(descs))(*descs)
        whole = L.qlora_linear_fwd_grouped_workspace(M, len(descs), arr)
        parts = []
        for i in range(0, len(descs), 8):
            sub = (q._LinearDesc * len(descs[i:i + 8]))(*descs[i:i + 8])
            parts.append(L.qlora_linear_fwd_grouped_workspace(M, len(descs[i:i + 8]), sub))
        assert whole == max(parts)
        one = (q._LinearDesc * 1)(descs[0])
        assert L.qlora_linear_fwd_grouped_workspace(M, 1, one) == L.qlora_linear_fwd_workspace(M, 4096, 4096, 16)


def test_adamw_host_checks():
    # the optimizer step's argument checks run on the host (no GPU needed)
    L = q.lib()
    fake = 1 << 20
    h = q.AdamwHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 1)
    p = ctypes.c_void_p(fake)
    assert L.qlora_adamw_step(None, p, p, p, 16, ctypes.byref(h), None, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_step(p, p, p, ctypes.c_void_p(fake + 4), 16, ctypes.byref(h), None, None) == \
        q.QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_step(p, p, p, p, 0, ctypes.byref(h), None, None) == q.QLORA_ERR_INVALID_ARG
    for bad in (q.AdamwHparams(1e-3, 0.9, 0.999, 1e-8, 0.0, 0), q.AdamwHparams(1e-3, 1.0, 0.999, 1e-8, 0.0, 1),
                q.AdamwHparams(float("nan"), 0.9, 0.999, 1e-8, 0.0, 1), q.AdamwHparams(1e-3, 0.9, 0.999, -1.0, 0.0, 1)):
        assert L.qlora_adamw_step(p, p, p, p, 16, ctypes.byref(bad), None, None) == q.QLORA_ERR_INVALID_ARG
    assert L.qlora_adamw_prefetch(None, 16, 1, None) == q.QLORA_ERR_INVALID_ARG
