"""GPU parity of the adapter's optimizer step (AdamW, the page's "update LoRA with a
paged optimizer", section 3; state in unified memory, section 2) against the oracle:
parameters, both moments and the bf16 adapter copy must match bit for bit after every
step, with the state in device memory and in managed memory paged out to the host
between steps."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_double_b200 as q
import oracle

pytestmark = pytest.mark.gpu


def _grads(n, steps, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return [(torch.randn(n, generator=g) * 1e-3 * (10.0 ** (s % 3 - 1))).float() for s in range(steps)]


def _check(theta, m, v, tb, th_ref, m_ref, v_ref, bits_ref):
    torch.cuda.synchronize()
    assert np.array_equal(theta.cpu().numpy().view(np.uint32), th_ref.view(np.uint32)), "theta"
    assert np.array_equal(m.cpu().numpy().view(np.uint32), m_ref.view(np.uint32)), "m"
    assert np.array_equal(v.cpu().numpy().view(np.uint32), v_ref.view(np.uint32)), "v"
    assert np.array_equal(tb.view(torch.int16).cpu().numpy().view(np.uint16), bits_ref), "bf16 copy"


@pytest.mark.parametrize("n", [1, 7, 4096 * 64 + 64 * 4096, (1 << 20) + 3])
@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_device_memory(n, wd):
    lr, b1, b2, eps = 2e-3, 0.9, 0.999, 1e-8
    theta0 = (torch.randn(n, generator=torch.Generator().manual_seed(n)) * 0.02).float()
    theta, m, v = theta0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    tb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    th_ref, m_ref, v_ref = theta0.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t, g in enumerate(_grads(n, 4, 11 + n), start=1):
        q.qlora_adamw_step(theta, g.cuda(), m, v, t, lr, b1, b2, eps, wd, theta_bf16=tb)
        bits = oracle.adamw_step(th_ref, g.numpy(), m_ref, v_ref, t, lr, b1, b2, eps, wd, want_bf16=True)
        assert q.qlora_get_device_status() == q.QLORA_OK
        _check(theta, m, v, tb, th_ref, m_ref, v_ref, bits)


def test_adamw_managed_state_paged_between_steps():
    # the paged setting: parameters and moments in managed memory, moved back to host
    # memory after every step and brought to the GPU again (explicitly, or by the step
    # touching them) before the next one
    n, lr, wd = (1 << 21) + 5, 1e-3, 0.02
    theta0 = (torch.randn(n, generator=torch.Generator().manual_seed(3)) * 0.02).float()
    theta, m, v = q.managed_empty(n), q.managed_empty(n), q.managed_empty(n)
    tb = q.managed_empty(n, torch.bfloat16)
    theta.copy_(theta0.cuda())
    m.zero_()
    v.zero_()
    th_ref, m_ref, v_ref = theta0.numpy().copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t, g in enumerate(_grads(n, 5, 99), start=1):
        if t % 2 == 0:
            for x in (theta, m, v):
                q.qlora_adamw_prefetch(x, to_device=True)
        q.qlora_adamw_step(theta, g.cuda(), m, v, t, lr, 0.9, 0.999, 1e-8, wd, theta_bf16=tb)
        for x in (theta, m, v, tb):
            q.qlora_adamw_prefetch(x, to_device=False)
        bits = oracle.adamw_step(th_ref, g.numpy(), m_ref, v_ref, t, lr, 0.9, 0.999, 1e-8, wd, want_bf16=True)
        assert q.qlora_get_device_status() == q.QLORA_OK
        _check(theta, m, v, tb, th_ref, m_ref, v_ref, bits)


def test_adamw_steps_the_layer_gradients():
    # the loop of the page's section 3 on a small layer: forward, backward, then one AdamW
    # step on dA and dB laid out back to back; the new bf16 adapter copy feeds the next forward
    import synth_inputs as si
    wl = si.workload("tiny")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0, device="cuda")
    t = q.qlora_nf4_quantize(inp["W"])
    na, nb = L.d_in * L.r, L.r * L.d_out
    theta = torch.cat([inp["A"].float().ravel(), inp["B"].float().ravel()])
    m, v = torch.zeros_like(theta), torch.zeros_like(theta)
    tb = torch.empty(na + nb, dtype=torch.bfloat16, device="cuda")
    th_ref, m_ref, v_ref = theta.cpu().numpy().copy(), np.zeros(na + nb, np.float32), np.zeros(na + nb, np.float32)
    A, B = inp["A"], inp["B"]
    for step in range(1, 4):
        Y, XA = q.qlora_linear_fwd(inp["X"], t, A, B, L.s)
        _, dA, dB = q.qlora_linear_bwd(inp["X"], inp["dY"], t, A, B, L.s, XA=XA)
        grad = torch.cat([dA.ravel(), dB.ravel()])
        q.qlora_adamw_step(theta, grad, m, v, step, 1e-3, theta_bf16=tb)
        bits = oracle.adamw_step(th_ref, grad.cpu().numpy(), m_ref, v_ref, step, 1e-3, want_bf16=True)
        _check(theta, m, v, tb, th_ref, m_ref, v_ref, bits)
        A, B = tb[:na].view(L.d_in, L.r), tb[na:].view(L.r, L.d_out)
    assert q.qlora_get_device_status() == q.QLORA_OK
