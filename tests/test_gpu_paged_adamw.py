"""GPU parity of the fused AdamW step against the oracle, one step at a time from the kernel's own fp32
state, in device memory and in managed memory (resident or evicted to the host between steps), and the
PagedAdamW optimizer on QLoRA layers."""
import numpy as np
import pytest
import torch

from oracle.adamw import adamw_step as oracle_step
import synth

pytestmark = pytest.mark.gpu


def f32(x):
    """The value the library receives for a float argument."""
    return float(np.float32(x))


def oracle(p, g, m, v, t, lr, wd):
    """The oracle step with the hyper-parameters as the fp32 values the kernel is given."""
    return oracle_step(p, g, m, v, t, f32(lr), beta1=f32(0.9), beta2=f32(0.999), eps=f32(1e-8), wd=f32(wd))


def _bounds_ok(p_new, m_new, v_new, ref, p_old, g, m_old, v_old, t, lr):
    """fp32 evaluation of one step against the exact fp64 step from the same fp32 inputs: a few roundings
    of each term (m may cancel, so its bound is on the terms, not on the sum)."""
    rp, rm, rv = ref
    e = 2.0 ** -22
    g, m_old, v_old = (np.asarray(a, np.float64) for a in (g, m_old, v_old))
    m_terms = 0.9 * np.abs(m_old) + 0.1 * np.abs(g)
    assert np.all(np.abs(m_new - rm) <= e * m_terms + 1e-38), "m"
    assert np.all(np.abs(v_new - rv) <= e * np.abs(rv) + 1e-38), "v"
    denom = np.sqrt(rv / (1 - 0.999 ** t)) + 1e-8
    upd_terms = lr * m_terms / (1 - 0.9 ** t) / denom
    assert np.all(np.abs(p_new - rp) <= e * np.abs(p_old) + 8 * e * upd_terms + 1e-38), "p"


def _run_steps(lib, n, steps, wd, make_state, evict=False):
    dev = torch.device("cuda", 0)
    p = torch.from_numpy(synth.normal_f32(n, 0.02, 21, 1)).to(dev)
    m, v = make_state(n), make_state(n)
    m.zero_(); v.zero_()
    p16 = torch.empty(n, dtype=torch.bfloat16, device=dev)
    hist = []
    for t in range(1, steps + 1):
        g = torch.from_numpy(synth.normal_f32(n, 1e-3 * t, 21, 100 + t)).to(dev)
        p0, m0, v0 = p.cpu().numpy().copy(), m.cpu().numpy().copy(), v.cpu().numpy().copy()
        if evict:
            lib.paged_prefetch(m, False)
            lib.paged_prefetch(v, False)
        lr = 2e-4 * (1 + 0.5 * (t % 2))
        lib.adamw_step(p, g, m, v, t, lr, weight_decay=wd, p_bf16=p16)
        torch.cuda.synchronize()
        pn, mn, vn = p.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy()
        gn = g.cpu().numpy()
        ref = oracle(p0, gn, m0, v0, t, lr, wd)
        _bounds_ok(pn, mn, vn, ref, p0, gn, m0, v0, t, lr)
        assert torch.equal(p16.cpu(), p.cpu().to(torch.bfloat16)), "bf16 copy"
        hist.append((pn.copy(), mn.copy(), vn.copy()))
    return hist


@pytest.mark.parametrize("n", [1, 3, 4, 5, 1000, (1 << 20) + 3])
@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_adamw_step_matches_the_oracle(lib, n, wd):
    _run_steps(lib, n, 4, wd, lambda k: torch.empty(k, dtype=torch.float32, device="cuda"))


def test_managed_states_give_the_same_bits_resident_or_evicted(lib):
    n = (1 << 22) + 7
    dev_hist = _run_steps(lib, n, 3, 0.05, lambda k: torch.empty(k, dtype=torch.float32, device="cuda"))
    res_hist = _run_steps(lib, n, 3, 0.05, lambda k: lib.paged_empty(k))
    ev_hist = _run_steps(lib, n, 3, 0.05, lambda k: lib.paged_empty(k), evict=True)
    for a, b, c in zip(dev_hist, res_hist, ev_hist):
        for x, y, z in zip(a, b, c):
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
            assert np.array_equal(x.view(np.uint32), z.view(np.uint32))


def test_paged_adamw_on_qlora_layers(lib):
    from bit_nf4_quantized_14_b200.autograd import QLoRALinear
    from bit_nf4_quantized_14_b200.optim import PagedAdamW
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    l1 = QLoRALinear(torch.randn(256, 128, device=dev, generator=gen) * 0.05, r=16, alpha=16, generator=gen)
    l2 = QLoRALinear(torch.randn(64, 256, device=dev, generator=gen) * 0.05, r=16, alpha=16, generator=gen)
    with torch.no_grad():
        l1.B.normal_(0, 0.01, generator=gen)
        l2.B.normal_(0, 0.01, generator=gen)
    params = [l1.A, l1.B, l2.A, l2.B]
    opt = PagedAdamW(params, lr=1e-3, weight_decay=0.01)
    x = torch.randn(40, 128, device=dev, generator=gen).to(torch.bfloat16)
    target = torch.randn(40, 64, device=dev, generator=gen)
    losses = []
    m = np.zeros(opt.n)
    v = np.zeros(opt.n)
    for t in range(1, 6):
        opt.zero_grad()
        if t == 3:
            opt.evict_states()
        if t == 4:
            opt.prefetch_states_async(evict_first=True)
        loss = ((l2(l1(x)).float() - target) ** 2).mean()
        loss.backward()
        p0 = opt.flat_p.cpu().numpy().copy()
        g = opt.flat_g.cpu().numpy().copy()
        m0, v0 = opt.m.cpu().numpy().copy(), opt.v.cpu().numpy().copy()
        assert np.any(g != 0)
        opt.step()
        torch.cuda.synchronize()
        ref = oracle(p0, g, m0, v0, t, 1e-3, 0.01)
        _bounds_ok(opt.flat_p.cpu().numpy(), opt.m.cpu().numpy(), opt.v.cpu().numpy(), ref, p0, g, m0, v0, t, 1e-3)
        # the parameters the layers see are the updated flat buffer
        assert torch.equal(l2.B.detach().reshape(-1).cpu(), opt.flat_p[-l2.B.numel():].cpu())
        losses.append(float(loss.detach()))
    assert losses[-1] < losses[0]
