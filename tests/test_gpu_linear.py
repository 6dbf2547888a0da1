"""GPU parity of the QLoRA linear forward and backward against the fp64 oracle.

Tolerance (stated for the layer): for each of Y, dX, dA, dB separately,
max|err| / max|ref| <= 2e-2 and ||err||_F / ||ref||_F <= 5e-3, where the
reference is the exact (fp64) product of the same bf16 operands and the
oracle's bf16 dequantised weight."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import oracle
import synth_inputs as si

pytestmark = pytest.mark.gpu

MAX_TOL = 2e-2
FRO_TOL = 5e-3
DEFAULT_PAIR_MIN_M = 128   # the library's default token count for the pair-GEMM route


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def check(got, ref, name):
    m, f = oracle.rel_errors(got, ref)
    assert m <= MAX_TOL and f <= FRO_TOL, f"{name}: max-rel {m:.3e}, fro-rel {f:.3e}"


def make_problem(M, rows, cols, r, seed, w_std=0.02, a_std=0.02, b_std=0.02, outliers=0.0):
    L = si.Layer("p", rows, cols, w_std, r=r, alpha=2.0 * r if r else 0.0, a_std=a_std, b_std=b_std,
                 outlier_frac=outliers)
    W = si.weight(L, seed, device="cuda")
    X = si.normal((M, cols), 1.0, seed + 1, device="cuda", dtype=torch.bfloat16)
    dY = si.normal((M, rows), 1.0, seed + 2, device="cuda", dtype=torch.bfloat16)
    A = si.normal((cols, r), a_std, seed + 3, device="cuda", dtype=torch.bfloat16) if r else None
    B = si.normal((r, rows), b_std, seed + 4, device="cuda", dtype=torch.bfloat16) if r else None
    return W, X, dY, A, B, (L.s if r else 0.0)


def oracle_weight(W):
    ref = oracle.quantize(W.float().cpu().numpy())
    return oracle.bf16_bits_to_f32(oracle.dequant(ref)).reshape(W.shape).astype(np.float64)


def run_case(M, rows, cols, r, seed, do_bwd=True, sample_rows=None, **kw):
    W, X, dY, A, B, s = make_problem(M, rows, cols, r, seed, **kw)
    t = q.qlora_nf4_quantize(W)
    Y, XA = q.qlora_linear_fwd(X, t, A, B, s)
    if do_bwd:
        dX, dA, dB = q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA)
    assert q.qlora_get_device_status() == q.QLORA_OK
    Wh = oracle_weight(W)
    Xn, dYn = f64(X), f64(dY)
    An = f64(A) if r else np.zeros((cols, 0))
    Bn = f64(B) if r else np.zeros((0, rows))
    idx = np.arange(M) if sample_rows is None else sample_rows
    Yref = oracle.linear_fwd(Xn[idx], Wh, An, Bn, s)
    check(f64(Y)[idx], Yref, "Y")
    if r:
        check(f64(XA)[idx], Xn[idx] @ An, "XA")
    if do_bwd:
        if sample_rows is None:
            dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wh, An, Bn, s)
        else:
            dXr, _, _ = oracle.linear_bwd(Xn[idx], dYn[idx], Wh, An, Bn, s)
            dAr, dBr = oracle.adapter_grads(Xn, dYn, An, Bn, s)
        check(f64(dX)[idx], dXr, "dX")
        if r:
            check(f64(dA), dAr, "dA")
            check(f64(dB), dBr, "dB")
    return Y


def test_tiny_layer():
    # 256 -> 512, 32 tokens, rank 8, alpha 16
    wl = si.workload("tiny")
    inp = si.layer_inputs(wl, 0, device="cuda")
    L = wl.layers[0]
    t = q.qlora_nf4_quantize(inp["W"])
    Y, XA = q.qlora_linear_fwd(inp["X"], t, inp["A"], inp["B"], L.s)
    dX, dA, dB = q.qlora_linear_bwd(inp["X"], inp["dY"], t, inp["A"], inp["B"], L.s, XA=XA)
    assert q.qlora_get_device_status() == q.QLORA_OK
    Wh = oracle_weight(inp["W"])
    Xn, dYn, An, Bn = (f64(inp[k]) for k in ("X", "dY", "A", "B"))
    check(f64(Y), oracle.linear_fwd(Xn, Wh, An, Bn, L.s), "Y")
    dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wh, An, Bn, L.s)
    check(f64(dX), dXr, "dX")
    check(f64(dA), dAr, "dA")
    check(f64(dB), dBr, "dB")


@pytest.mark.parametrize("M,rows,cols,r", [
    (300, 400, 320, 24),     # several tiles in every dimension, ragged tails, r % 16 != 0
    (300, 400, 320, 0),      # no adapter
    (257, 272, 192, 64),
    (520, 384, 640, 128),    # two adapter K blocks
    (17, 128, 128, 16),      # just above the small-M path
    (1000, 1024, 1088, 8),
])
def test_multi_tile_ragged(M, rows, cols, r):
    run_case(M, rows, cols, r, seed=M + rows + cols + r)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("r", [0, 16])
def test_small_m_gemv(M, r):
    run_case(M, 1024, 2048 + 64, r, seed=100 + M + r)


@pytest.mark.parametrize("M,rows,cols,r", [
    (3, 400, 320, 24),       # rows past the last 32-row block, one partial K chunk
    (5, 48, 4096, 16),       # odd M, two K chunks, a half row block
    (8, 4096, 11008, 16),    # the long-K projection: six chunks, the last 768 inputs
    (16, 272, 192, 64),
    (1, 16, 64, 8),          # a single 64-block
    (9, 1040, 4160, 256),    # widest adapter, ragged rows and K chunks
    (12, 2064, 1600, 0),
])
def test_small_m_ragged(M, rows, cols, r):
    # the forward at these sizes runs the small-M kernels; the backward the GEMM path
    run_case(M, rows, cols, r, seed=7 * M + rows + cols + r, do_bwd=r <= 128)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_layer_full(M):
    # one Llama-7B-shaped block at decode sizes, forward only (rank 16 on q, k, v, o)
    wl = si.workload("decode7b", M=M)
    for li, L in enumerate(wl.layers):
        inp = si.layer_inputs(wl, li, device="cuda")
        t = q.qlora_nf4_quantize(inp["W"])
        Y, _ = q.qlora_linear_fwd(inp["X"], t, inp.get("A"), inp.get("B"), L.s)
        assert q.qlora_get_device_status() == q.QLORA_OK
        Wh = oracle_weight(inp["W"])
        An = f64(inp["A"]) if L.r else np.zeros((L.d_in, 0))
        Bn = f64(inp["B"]) if L.r else np.zeros((0, L.d_out))
        check(f64(Y), oracle.linear_fwd(f64(inp["X"]), Wh, An, Bn, L.s), f"Y[{L.name}]")


@pytest.mark.parametrize("M", [1, 16])
def test_decode_layer_grouped(M):
    # the whole block in one grouped call, every projection against the oracle. Each output
    # row sums its K slices in slice order and its K chunks in chunk order whichever CTA holds
    # them, so the grouped call is bit-identical to the single calls and to itself.
    wl = si.workload("decode7b", M=M)
    items, singles, refs = [], [], []
    for li, L in enumerate(wl.layers):
        inp = si.layer_inputs(wl, li, device="cuda")
        t = q.qlora_nf4_quantize(inp["W"])
        xa = torch.empty(M, L.r, dtype=torch.bfloat16, device="cuda") if L.r else None
        items.append({"X": inp["X"], "W": t, "A": inp.get("A"), "B": inp.get("B"), "s": L.s, "XA_save": xa})
        Ys, XAs = q.qlora_linear_fwd(inp["X"], t, inp.get("A"), inp.get("B"), L.s)
        singles.append((Ys, XAs))
        Wh = oracle_weight(inp["W"])
        An = f64(inp["A"]) if L.r else np.zeros((L.d_in, 0))
        Bn = f64(inp["B"]) if L.r else np.zeros((0, L.d_out))
        refs.append(oracle.linear_fwd(f64(inp["X"]), Wh, An, Bn, L.s))
    Ys = [y.clone() for y in q.qlora_linear_fwd_grouped(items)]
    Ys2 = q.qlora_linear_fwd_grouped(items)
    assert q.qlora_get_device_status() == q.QLORA_OK
    for li, ((Y1, XA1), Yg, Yg2, it) in enumerate(zip(singles, Ys, Ys2, items)):
        name = wl.layers[li].name
        check(f64(Yg), refs[li], f"Y[{name}]")
        assert torch.equal(Yg, Yg2), name
        assert torch.equal(Yg, Y1), name
        if XA1 is not None:
            assert torch.equal(XA1, it["XA_save"])


@pytest.mark.parametrize("M", [2, 8, 9])
def test_grouped_more_than_eight(M):
    # eleven projections of mixed shapes: two launch groups (eight, then three) that share
    # one workspace; ragged rows (N % 32 == 16), inputs that end inside a K chunk and a slice
    shapes = [(48, 4096, 16), (16, 64, 8), (400, 320, 24), (1040, 4160, 0), (272, 2112, 64), (32, 2048, 8),
              (2064, 1600, 0), (128, 6144, 16), (80, 576, 0), (16, 2048, 256), (96, 4224, 8)]
    items, refs = [], []
    for i, (rows, cols, r) in enumerate(shapes):
        W, X, dY, A, B, s = make_problem(M, rows, cols, r, seed=900 + 13 * i + M)
        t = q.qlora_nf4_quantize(W)
        xa = torch.empty(M, r, dtype=torch.bfloat16, device="cuda") if r else None
        items.append({"X": X, "W": t, "A": A, "B": B, "s": s, "XA_save": xa})
        An = f64(A) if r else np.zeros((cols, 0))
        Bn = f64(B) if r else np.zeros((0, rows))
        refs.append((oracle.linear_fwd(f64(X), oracle_weight(W), An, Bn, s), f64(X) @ An))
    Ys = q.qlora_linear_fwd_grouped(items)
    assert q.qlora_get_device_status() == q.QLORA_OK
    for i, (Y, it, (ref, xaref)) in enumerate(zip(Ys, items, refs)):
        check(f64(Y), ref, f"Y[{i}]")
        if it["XA_save"] is not None:
            check(f64(it["XA_save"]), xaref, f"XA[{i}]")
        Y1, _ = q.qlora_linear_fwd(it["X"], it["W"], it["A"], it["B"], it["s"])
        assert torch.equal(Y, Y1), i


@pytest.mark.parametrize("M,rows,cols,r", [(3, 400, 320, 24), (100, 272, 640, 64), (200, 272, 640, 64),
                                           (1024, 512, 1024, 16)])
def test_backward_recomputes_xa(M, rows, cols, r):
    # XA = NULL: the backward recomputes X A itself (small-M, fused (M = 100) and CTA-pair
    # paths)
    W, X, dY, A, B, s = make_problem(M, rows, cols, r, seed=31 * M + rows)
    t = q.qlora_nf4_quantize(W)
    dX, dA, dB = q.qlora_linear_bwd(X, dY, t, A, B, s, XA=None)
    assert q.qlora_get_device_status() == q.QLORA_OK
    Wh = oracle_weight(W)
    dXr, dAr, dBr = oracle.linear_bwd(f64(X), f64(dY), Wh, f64(A), f64(B), s)
    check(f64(dX), dXr, "dX")
    check(f64(dA), dAr, "dA")
    check(f64(dB), dBr, "dB")


def test_full_4096_layer_sampled():
    # the 4096 x 4096 layer at 4096 tokens, rank 64, in the bench's launch configuration
    M = 4096
    rows_idx = np.unique(np.concatenate([[0, 1, 255, 256, M - 1], np.random.default_rng(0).integers(0, M, 60)]))
    wl = si.workload("l4096")
    inp = si.layer_inputs(wl, 0, device="cuda")
    L = wl.layers[0]
    t = q.qlora_nf4_quantize(inp["W"])
    Y, XA = q.qlora_linear_fwd(inp["X"], t, inp["A"], inp["B"], L.s)
    dX, dA, dB = q.qlora_linear_bwd(inp["X"], inp["dY"], t, inp["A"], inp["B"], L.s, XA=XA)
    assert q.qlora_get_device_status() == q.QLORA_OK
    Wh = oracle_weight(inp["W"])
    Xn, dYn, An, Bn = (f64(inp[k]) for k in ("X", "dY", "A", "B"))
    check(f64(Y)[rows_idx], oracle.linear_fwd(Xn[rows_idx], Wh, An, Bn, L.s), "Y")
    dXr, _, _ = oracle.linear_bwd(Xn[rows_idx], dYn[rows_idx], Wh, An, Bn, L.s)
    check(f64(dX)[rows_idx], dXr, "dX")
    dAr, dBr = oracle.adapter_grads(Xn, dYn, An, Bn, L.s)
    check(f64(dA), dAr, "dA")
    check(f64(dB), dBr, "dB")


def test_70b_projections_sampled():
    # two projections of the 70B-like block at 4096 tokens: the skinny-N k projection
    # and the long-K down projection
    wl = si.workload("l70b")
    M = 4096
    rows_idx = np.array([0, 1, 1000, 2047, 2048, 4095])
    for name in ("k", "down"):
        li = [l.name for l in wl.layers].index(name)
        L = wl.layers[li]
        inp = si.layer_inputs(wl, li, device="cuda")
        t = q.qlora_nf4_quantize(inp["W"])
        Y, XA = q.qlora_linear_fwd(inp["X"], t, inp["A"], inp["B"], L.s)
        dX, dA, dB = q.qlora_linear_bwd(inp["X"], inp["dY"], t, inp["A"], inp["B"], L.s, XA=XA)
        assert q.qlora_get_device_status() == q.QLORA_OK
        Wh = oracle_weight(inp["W"])
        Xn, dYn, An, Bn = (f64(inp[k]) for k in ("X", "dY", "A", "B"))
        check(f64(Y)[rows_idx], oracle.linear_fwd(Xn[rows_idx], Wh, An, Bn, L.s), f"Y[{name}]")
        dXr, _, _ = oracle.linear_bwd(Xn[rows_idx], dYn[rows_idx], Wh, An, Bn, L.s)
        check(f64(dX)[rows_idx], dXr, f"dX[{name}]")
        dAr, dBr = oracle.adapter_grads(Xn, dYn, An, Bn, L.s)
        check(f64(dA), dAr, f"dA[{name}]")
        check(f64(dB), dBr, f"dB[{name}]")
        del inp, t, Y, XA, dX, dA, dB, Wh, Xn, dYn
        torch.cuda.empty_cache()


def test_zero_adapter_equals_plain_product():
    # B = 0 (or s = 0) leaves the plain dequantised product, checked against
    # torch.matmul on the dequantised weight
    W, X, dY, A, B, s = make_problem(384, 256, 512, 16, seed=77)
    t = q.qlora_nf4_quantize(W)
    Wh = q.qlora_nf4_dequant(t)
    Y0, _ = q.qlora_linear_fwd(X, t, A, torch.zeros_like(B), s)
    Y1, _ = q.qlora_linear_fwd(X, t, A, B, 0.0)
    ref = torch.matmul(X.double(), Wh.double().T)
    for Y in (Y0, Y1):
        m, f = oracle.rel_errors(f64(Y), ref.cpu().numpy())
        assert m <= MAX_TOL and f <= FRO_TOL


@pytest.mark.parametrize("M,rows,cols,r", [
    (512, 512, 8192, 64),     # forward: 4 tiles, 16 K ranges per tile; dgrad: 64 whole tiles
    (200, 384, 2048, 64),     # 200 tokens: one 256-token tile, 2 and 8 output tiles
    (4096, 256, 4096, 16),    # headline tokens, a narrow output: 16 tiles, 4 K ranges
])
def test_split_k_pair_route(M, rows, cols, r):
    # few output tiles: the pair GEMM splits each tile's K blocks over the idle SMs and adds
    # the fp32 partials in a fixed order; every element against the oracle
    run_case(M, rows, cols, r, seed=M + rows + cols)


@pytest.mark.parametrize("rep", [0, 1])
def test_many_tiles_per_cta_fused_full(rep):
    # with the pair route raised to 512 tokens: at 480 the forward of the 16384-row weight
    # and the dgrad of the 16384-input one stay on the fused kernels, where every persistent
    # CTA walks several 128 x 256 tiles; the other two directions have 16 fused tiles and
    # take the pair GEMM with split K. Compare every element, twice, so a race at tile
    # boundaries shows
    M = 480
    for rows, cols in ((16384, 1024), (1024, 16384)):
        W, X, dY, A, B, s = make_problem(M, rows, cols, 64, seed=500 + rows + rep)
        t = q.qlora_nf4_quantize(W)
        q.lib().qlora_linear_set_pair_min_m(512)
        try:
            Y, XA = q.qlora_linear_fwd(X, t, A, B, s)
            dX, dA, dB = q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA)
        finally:
            q.lib().qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)
        assert q.qlora_get_device_status() == q.QLORA_OK
        Wh = oracle_weight(W)
        Xn, dYn, An, Bn = f64(X), f64(dY), f64(A), f64(B)
        check(f64(Y), oracle.linear_fwd(Xn, Wh, An, Bn, s), f"Y[{rows}x{cols}]")
        dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wh, An, Bn, s)
        check(f64(dX), dXr, f"dX[{rows}x{cols}]")
        check(f64(dA), dAr, f"dA[{rows}x{cols}]")
        check(f64(dB), dBr, f"dB[{rows}x{cols}]")


@pytest.mark.parametrize("rep", [0, 1])
def test_many_tiles_per_cta_full(rep):
    # at 4096 tokens the CTA-pair GEMM runs; here the forward of the 8192-row
    # weight and the dgrad of the 8192-input one give each pair about seven 256 x 256
    # tiles, so both TMEM accumulators are reused many times: compare every element,
    # twice, so a race between the epilogue and the next tile's MMAs shows
    M = 4096
    for rows, cols in ((1024, 8192), (8192, 1024)):
        W, X, dY, A, B, s = make_problem(M, rows, cols, 64, seed=300 + rows + rep)
        t = q.qlora_nf4_quantize(W)
        Y, XA = q.qlora_linear_fwd(X, t, A, B, s)
        dX, dA, dB = q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA)
        assert q.qlora_get_device_status() == q.QLORA_OK
        Wh = oracle_weight(W)
        Xn, dYn, An, Bn = f64(X), f64(dY), f64(A), f64(B)
        check(f64(Y), oracle.linear_fwd(Xn, Wh, An, Bn, s), f"Y[{rows}x{cols}]")
        dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wh, An, Bn, s)
        check(f64(dX), dXr, f"dX[{rows}x{cols}]")
        check(f64(dA), dAr, f"dA[{rows}x{cols}]")
        check(f64(dB), dBr, f"dB[{rows}x{cols}]")


@pytest.mark.parametrize("P,M,rows,cols,r", [
    (2 ** 63 - 1, 1024, 512, 1024, 16),   # the fused dequant-GEMM at four token tiles
    (2 ** 63 - 1, 4096, 256, 512, 64),    # ... and at the headline's 4096 tokens
    (17, 100, 400, 320, 24),          # the dequant + CTA-pair route below one 256-token tile
    (17, 300, 272, 192, 64),
])
def test_routes_forced_either_way(P, M, rows, cols, r):
    # both large-M routes compute the same layer at any token count
    q.lib().qlora_linear_set_pair_min_m(P)
    try:
        run_case(M, rows, cols, r, seed=M + rows + r + 7)
    finally:
        q.lib().qlora_linear_set_pair_min_m(DEFAULT_PAIR_MIN_M)


@pytest.mark.parametrize("M,rows,cols,r", [(512, 1024, 2048, 16), (600, 768, 1536, 0), (256, 4096, 1024, 8),
                                           (4096, 1024, 4096, 16), (4096, 2048, 1024, 16)])
def test_workspace_weight_bit_exact(M, rows, cols, r):
    # On the pair route the layer dequantises the weight into its workspace, which starts
    # with the adapter scratch (forward: s XA, M x r bf16; backward: s G and X A), each
    # rounded up to 256 bytes, followed by the bf16 weight: after the call that weight must
    # equal the oracle's dequantisation bit for bit, and the layer's outputs stay within the
    # tolerance. The dequantisation runs as its own kernel on a second stream, or inside the
    # adapter product before the GEMM when that product has one CTA on most SMs and K >= 2048:
    # the two M = 4096 cases take that route in the forward (K = 4096) and in the backward
    # (K = d_out = 2048).
    W, X, dY, A, B, s = make_problem(M, rows, cols, r, 7100 + M + r)
    t = q.qlora_nf4_quantize(W)
    L = q.lib()
    mr = ((M * r * 2 + 255) // 256) * 256 if r else 0
    want = oracle.dequant(oracle.quantize(W.float().cpu().numpy())).reshape(rows, cols)
    ws_f = torch.zeros(L.qlora_linear_fwd_workspace(M, rows, cols, r), dtype=torch.uint8, device="cuda")
    Y, XA = q.qlora_linear_fwd(X, t, A, B, s, ws=ws_f)
    ws_b = torch.zeros(L.qlora_linear_bwd_workspace(M, rows, cols, r), dtype=torch.uint8, device="cuda")
    dX, dA, dB = q.qlora_linear_bwd(X, dY, t, A, B, s, XA=XA, ws=ws_b)
    torch.cuda.synchronize()
    assert q.qlora_get_device_status() == q.QLORA_OK
    n = rows * cols * 2
    if M >= 512:
        got_f = ws_f[mr:mr + n].view(torch.int16).cpu().numpy().view(np.uint16).reshape(rows, cols)
        assert np.array_equal(got_f, want), "forward workspace weight"
    got_b = ws_b[2 * mr:2 * mr + n].view(torch.int16).cpu().numpy().view(np.uint16).reshape(rows, cols)
    assert np.array_equal(got_b, want), "backward workspace weight"
    Wh = oracle_weight(W)
    Xn, dYn = f64(X), f64(dY)
    An = f64(A) if r else np.zeros((cols, 0))
    Bn = f64(B) if r else np.zeros((0, rows))
    check(f64(Y), oracle.linear_fwd(Xn, Wh, An, Bn, s), "Y")
    dXr, dAr, dBr = oracle.linear_bwd(Xn, dYn, Wh, An, Bn, s)
    check(f64(dX), dXr, "dX")
    if r:
        check(f64(dA), dAr, "dA")
        check(f64(dB), dBr, "dB")
