"""GPU vs oracle: the adapter optimiser step (AdamW) whose states the QLoRA page pages
between device and host memory (aizip.shop/methodologies/qlora, section "3. Paged
Optimizer").

The fp32 step is compared with the fp64 oracle over five steps: theta within
1e-6 |theta| + 1e-5 lr, m and v within 1e-5 relative (plus a floor), the bf16 copy equal
to the rounding of the kernel's own theta and, as a value, within one bf16 spacing of the
oracle's.
States held in paged (managed) memory and moved to the host between steps give
bit-identical results to device memory."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-3, beta1=0.9, beta2=0.995, eps=1e-8, weight_decay=0.01)


def _grads(n, steps, seed):
    return [synth.normal_bf16((n,), 1e-3 * (1 + t), seed, 60 + t).float() for t in range(steps)]


def _check(theta_g, m_g, v_g, p_g, theta_r, m_r, v_r, lr):
    th = theta_g.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(th - theta_r) <= 1e-6 * np.abs(theta_r) + 1e-5 * lr)
    for got, ref, nm in ((m_g, m_r, "m"), (v_g, v_r, "v")):
        g = got.cpu().numpy().astype(np.float64)
        floor = 1e-6 * np.max(np.abs(ref))
        assert np.all(np.abs(g - ref) <= 1e-5 * np.abs(ref) + floor), nm
    bits = p_g.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(bits, o.f32_to_bf16_bits(theta_g.cpu().numpy()))
    # against the oracle's rounding: one bf16 spacing (2^-7 relative at most) plus theta's
    # own tolerance, compared as values (near zero the bit patterns say nothing)
    got = o.bf16_bits_to_f32(bits).astype(np.float64)
    ref = o.bf16_bits_to_f32(o.f32_to_bf16_bits(theta_r.astype(np.float32))).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6 * np.abs(theta_r) + 1e-5 * lr)


@pytest.mark.parametrize("n", [4096 * 64, 1_000_003, 5, 1, 63, 65])
def test_adamw_matches_oracle(n):
    theta0 = synth.normal_bf16((n,), 0.02, 7, 59).float()
    grads = _grads(n, 5, 7)
    theta, m, v = theta0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    param = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    tr, mr, vr = theta0.numpy().astype(np.float64), np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        B.adamw_step(theta, param, g.cuda(), m, v, t, grad_scale=0.5, **HP)
        tr, mr, vr, _ = o.adamw_step(tr, g.numpy(), mr, vr, t, grad_scale=0.5, **HP)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    _check(theta, m, v, param, tr, mr, vr, HP["lr"])


def test_adamw_paged_states_match_device_states():
    """theta, m, v in paged memory, moved to the host between steps (so the step pages them
    back in), equal the same steps on device memory bit for bit; the host reads the states
    through the same pointer."""
    n = 300_000
    theta0 = synth.normal_bf16((n,), 0.02, 8, 59).float()
    grads = _grads(n, 3, 8)
    theta, m, v = theta0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    param = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    buf = B.PagedBuffer(3 * n * 4)
    pt, pm, pv = (buf.view(torch.float32, n, i * n * 4) for i in range(3))
    pt.copy_(theta0.cuda())
    pm.zero_()
    pv.zero_()
    pparam = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    for t, g in enumerate(grads, start=1):
        gd = g.cuda()
        B.adamw_step(theta, param, gd, m, v, t, **HP)
        buf.prefetch(to_host=True)
        B.adamw_step(pt, pparam, gd, pm, pv, t, **HP)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    for a, b in ((theta, pt), (m, pm), (v, pv)):
        assert torch.equal(a, b)
    assert torch.equal(param.view(torch.int16), pparam.view(torch.int16))
    buf.prefetch(to_host=True)
    torch.cuda.synchronize()
    host_m = buf.host_array(np.float32, n, n * 4)
    assert np.array_equal(host_m, m.cpu().numpy())
    buf.prefetch(to_host=False)
    torch.cuda.synchronize()
    del pt, pm, pv
    buf.free()


def test_adamw_nonfinite_gradient_is_flagged():
    n = 1024
    theta = torch.zeros(n, device="cuda")
    m, v = torch.zeros_like(theta), torch.zeros_like(theta)
    param = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(n, device="cuda")
    g[17] = float("inf")
    B.adamw_step(theta, param, g, m, v, 1, **HP)
    assert B.device_status() == B.QL_ERR_NONFINITE
    B.adamw_step(theta, param, torch.zeros_like(g), torch.zeros_like(m), torch.zeros_like(v), 1, **HP)
    assert B.device_status() == B.QL_OK


# ---- Lion with INT8 momentum (QFT page, section 2.1) -----------------------------------

@pytest.mark.parametrize("n", [64 * 4096, 1_000_003, 37, 1, 63, 65, 127])
def test_lion_int8_bit_exact(n):
    """Four steps: theta, the momentum codes and absmax, and the bf16 copy are bit-identical
    to the oracle (the step is fixed fp32 arithmetic; the codes are integer decisions)."""
    theta0 = synth.normal_bf16((n,), 0.02, 9, 59).float()
    grads = _grads(n, 4, 9)
    nb = (n + 63) // 64
    theta = theta0.cuda()
    codes = torch.zeros(n, dtype=torch.int8, device="cuda")
    amax = torch.zeros(nb, dtype=torch.float32, device="cuda")
    param = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    tr, cr, ar = theta0.numpy(), np.zeros(n, np.int8), np.zeros(nb, np.float32)
    hp = dict(lr=1e-4, beta1=0.9, beta2=0.99, weight_decay=0.1)
    for g in grads:
        B.lion_int8_step(theta, param, g.cuda(), codes, amax, **hp)
        tr, cr, ar, br = o.lion_int8_step(tr, g.numpy(), cr, ar, **hp)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    assert np.array_equal(theta.cpu().numpy().view(np.uint32), tr.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), cr)
    assert np.array_equal(amax.cpu().numpy().view(np.uint32), ar.view(np.uint32))
    assert np.array_equal(param.view(torch.int16).cpu().numpy().view(np.uint16), br)


def test_lion_int8_paged_states():
    """The INT8 momentum and theta in paged memory, moved to the host between steps, give
    the same bits as device memory."""
    n = 200_000
    nb = (n + 63) // 64
    theta0 = synth.normal_bf16((n,), 0.02, 10, 59).float()
    grads = _grads(n, 3, 10)
    buf = B.PagedBuffer(n * 4 + nb * 4 + n)
    pt = buf.view(torch.float32, n)
    pa = buf.view(torch.float32, nb, n * 4)
    pc = buf.view(torch.int8, n, n * 4 + nb * 4)
    pt.copy_(theta0.cuda())
    pa.zero_()
    pc.zero_()
    theta, codes = theta0.cuda(), torch.zeros(n, dtype=torch.int8, device="cuda")
    amax = torch.zeros(nb, device="cuda")
    p1 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    p2 = torch.empty_like(p1)
    for g in grads:
        gd = g.cuda()
        B.lion_int8_step(theta, p1, gd, codes, amax, 1e-4)
        buf.prefetch(to_host=True)
        B.lion_int8_step(pt, p2, gd, pc, pa, 1e-4)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    assert torch.equal(theta, pt) and torch.equal(codes, pc) and torch.equal(amax, pa)
    del pt, pa, pc
    buf.free()
