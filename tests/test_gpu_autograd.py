"""The autograd wrapper: QLoRALinear's forward and the gradients autograd delivers to x, A and B match the
oracle (the wrapper only marshals), and a small LLaMA-shaped decoder built from it trains (loss falls
over a few AdamW steps on a fixed batch)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu
TOL = 5e-3


def rel(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


@pytest.mark.parametrize("T", [3, 200])
def test_qlora_linear_module_matches_oracle(lib, T):
    from bit_nf4_quantized_14_b200.autograd import QLoRALinear
    N, K, r, alpha = 264, 320, 16, 16.0
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=alpha, seed=31)
    m = QLoRALinear(torch.from_numpy(case["W"]).cuda(), r=r, alpha=alpha)
    with torch.no_grad():                                   # adapters as bf16 values, so the oracle sees the same
        m.A.copy_(case["A"].float().cuda())
        m.B.copy_(case["B"].float().cuda())
    x = case["X"].cuda().requires_grad_(True)
    y = m(x)
    y.backward(case["dY"].cuda())
    Wt = O.bf16_bits_to_f32(O.dequantize(O.quantize(case["W"]), "bf16")).reshape(N, K)
    h = {k: synth.bf16_values(case[k]) for k in ("X", "A", "B", "dY")}
    Yr, _ = O.linear_fwd(h["X"], Wt, h["A"], h["B"], alpha)
    dXr, dAr, dBr = O.linear_bwd(h["dY"], h["X"], Wt, h["A"], h["B"], alpha)
    assert rel(y.detach().float().cpu(), Yr) <= TOL
    assert rel(x.grad.float().cpu(), dXr) <= TOL
    assert rel(m.A.grad.cpu(), dAr) <= TOL and rel(m.B.grad.cpu(), dBr) <= TOL
    assert m.A.grad.dtype == torch.float32 and m.B.grad.dtype == torch.float32


def test_small_decoder_trains(lib):
    import bench
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    model = bench.build_decoder(layers=2, d=256, ffn=512, heads=4, vocab=512, r=8, gen=gen, device=dev)
    params = [p for p in model.parameters() if p.requires_grad]
    assert len(params) == 2 * 7 * 2                       # A and B of the seven linears of two layers
    opt = torch.optim.AdamW(params, lr=1e-2, weight_decay=0.0)
    ids = torch.randint(0, 512, (64,), device=dev, generator=gen)
    tgt = torch.randint(0, 512, (64,), device=dev, generator=gen)
    losses = []
    for _ in range(12):
        loss = model(ids, tgt)
        loss.backward()
        opt.step()
        opt.zero_grad(set_to_none=True)
        losses.append(float(loss.item()))
    assert all(np.isfinite(losses)) and lib.get_status() == 0
    assert losses[-1] < losses[0] - 0.05, losses
