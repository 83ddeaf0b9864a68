"""GPU parity of the AdamW step on the adapters (qlora_adamw) and of the
paged (managed-memory) optimiser states.

The oracle is the fp64 AdamW step (Loshchilov and Hutter) applied to the
kernel's own fp32 state of the step before, so every step is checked against
one fp32 rounding budget: m and v to a few ulp, the parameter to a few ulp of
itself plus a few ulp of the step lr * m^/(sqrt(v^) + eps).  The bf16 copy is
bit-exact against round-to-nearest-even of the fp32 parameter.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200.optim import AdapterAdamW

pytestmark = pytest.mark.gpu
DEV = "cuda"
U32 = 2.0 ** -23


def _f32(hp):
    # the ABI takes fp32 hyper-parameters: the oracle gets the same values
    full = dict(beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, grad_scale=1.0) | hp
    return {k: float(np.float32(v)) for k, v in full.items()}


def _check_step(p0, g, m0, v0, t, hp, p, m, v, p16):
    hp = _f32(hp)
    pr, mr, vr = oracle.adamw_step(p0, g, m0, v0, t, **hp)
    b1, b2 = hp["beta1"], hp["beta2"]
    gg = np.abs(g.astype(np.float64) * hp["grad_scale"])
    # m may cancel: its error is a few ulp of the terms, not of the sum
    m_terms = np.abs(mr) + b1 * np.abs(m0) + (1 - b1) * gg
    assert np.all(np.abs(m - mr) <= 4 * U32 * m_terms + 1e-40)
    assert np.all(np.abs(v - vr) <= 4 * U32 * (np.abs(vr) + b2 * np.abs(v0) + (1 - b2) * gg * gg) + 1e-40)
    upd = hp["lr"] * (m_terms / (1 - b1 ** t) / (np.sqrt(vr / (1 - b2 ** t)) + hp["eps"])
                      + abs(hp["weight_decay"]) * np.abs(p0))
    err = np.abs(p - pr)
    bound = 2 * U32 * np.abs(pr) + 16 * U32 * upd + 1e-40
    assert np.all(err <= bound), float(np.max(err / bound))
    ref16 = torch.from_numpy(p.astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(p16.cpu().view(torch.int16), ref16.view(torch.int16))


HPARAMS = [
    dict(lr=1e-3),
    dict(lr=2e-4, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.01, grad_scale=1 / 1024),
    dict(lr=0.05, weight_decay=0.1, grad_scale=4.0),
]


@pytest.mark.parametrize("n", [1, 3, 4, 1029, 16 * 4096 + 64 * 16 + 16 * 4096 + 7,
                               3 * 2 ** 20 + 2])
@pytest.mark.parametrize("hi", range(len(HPARAMS)))
def test_adamw_against_oracle(n, hi):
    hp = HPARAMS[hi]
    gen = torch.Generator().manual_seed(n + 7 * hi)
    p = (torch.randn(n, generator=gen) * 0.05).to(DEV)
    m = torch.zeros(n, device=DEV)
    v = torch.zeros(n, device=DEV)
    p16 = torch.empty(n, dtype=torch.bfloat16, device=DEV)
    for t in range(1, 5):
        g = torch.randn(n, generator=gen) * (10.0 ** (-t))  # shrinking gradients
        if t == 3:
            g[::5] = 0.0
        state = [x.cpu().numpy().copy() for x in (p, m, v)]
        Q.qlora_adamw(p, g.to(DEV), m, v, t, param_bf16=p16, **hp)
        torch.cuda.synchronize()
        _check_step(state[0], g.numpy(), state[1], state[2], t, hp,
                    p.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy(), p16)


def test_adamw_empty_and_errors():
    z = torch.zeros(8, device=DEV)
    Q.qlora_adamw(z[:0], z[:0], z[:0], z[:0], 1, 1e-3)  # n = 0: nothing to do
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_adamw(z, z, z, z, 0, 1e-3)
    assert e.value.status == Q.QLORA_ERR_SHAPE
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_adamw(z[1:5], z[:4], z[:4], z[:4], 1, 1e-3)
    assert e.value.status == Q.QLORA_ERR_ALIGN
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_adamw(z, z, z, z, 1, 1e-3, beta2=1.0)
    assert e.value.status == Q.QLORA_ERR_UNSUPPORTED


def test_paged_states_match_device_states():
    # the same steps with moments in HBM and in managed memory sent to host
    # memory between steps: bit-identical results
    r, d_in, d_out = 16, 1024, 768
    gen = torch.Generator().manual_seed(5)
    A = (torch.randn(r, d_in, generator=gen) * 0.02).to(torch.bfloat16).to(DEV)
    B = (torch.randn(d_out, r, generator=gen) * 0.02).to(torch.bfloat16).to(DEV)
    opt_d = AdapterAdamW(A, B, lr=1e-3, weight_decay=0.01)
    opt_p = AdapterAdamW(A, B, lr=1e-3, weight_decay=0.01, paged=True)
    bucket = opt_d.grad_bucket()
    for _ in range(3):
        bucket.dA.copy_(torch.randn(r, d_in, generator=gen))
        bucket.dB.copy_(torch.randn(d_out, r, generator=gen))
        opt_d.step(bucket)
        opt_p.step(bucket)
        opt_p.offload()
        torch.cuda.synchronize()
    assert torch.equal(opt_d.master, opt_p.master)
    assert torch.equal(opt_d.m, opt_p.m.to(DEV)) and torch.equal(opt_d.v, opt_p.v.to(DEV))
    assert torch.equal(opt_d.A, opt_p.A) and torch.equal(opt_d.B, opt_p.B)
    # the bf16 views hold the rounded master weights at the GradBucket offsets
    assert torch.equal(opt_d.A, opt_d.master[:r * d_in].view(r, d_in).to(torch.bfloat16))
    off = bucket.off_b
    assert torch.equal(opt_d.B, opt_d.master[off:off + d_out * r].view(d_out, r).to(torch.bfloat16))


def test_training_step_moves_adapters_downhill():
    # forward, backward and AdamW on one layer, B starting at zero, towards
    # the output of the same layer with another B: 0.5 |Y - T|^2 falls
    from bit_nf4_quantized_17_b200 import workloads as WL
    shape = WL.LinearShape(512, 1024, 16, 32.0)
    inp = WL.linear_inputs(shape, 256, 11)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    X = inp["X"].to(DEV)
    A0 = inp["A"].to(DEV)
    B_target = WL.randn((512, 16), 0.05, 4, torch.bfloat16).to(DEV)
    T = Q.qlora_linear_fwd(q, A0, B_target, shape.alpha, X).float()
    opt = AdapterAdamW(A0, torch.zeros_like(B_target), lr=5e-3)
    bucket = opt.grad_bucket()
    U = torch.empty((256, 16), dtype=torch.float32, device=DEV)
    losses = []
    for _ in range(30):
        Y = Q.qlora_linear_fwd(q, opt.A, opt.B, shape.alpha, X, U_save=U)
        dY = Y.float() - T
        losses.append(0.5 * float((dY * dY).sum()))
        Q.qlora_linear_bwd(q, opt.A, opt.B, shape.alpha, X, U, dY.to(torch.bfloat16),
                           dA=bucket.dA, dB=bucket.dB, want_dx=False)
        opt.step(bucket)
    torch.cuda.synchronize()
    assert losses[-1] < 0.2 * losses[0], losses
