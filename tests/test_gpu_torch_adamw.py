"""The step of one rank against torch.optim.AdamW on the same fp32 gradients.

With R = 1 and fp32 gradients the fused step is plain AdamW on fp32
masters, which torch implements independently of this repository:
decoupled weight decay on the weight before the update, the bias-corrected
moments and eps outside the square root -- the same update, written the same
way.  Masters and moments must agree within the step's tolerance, and the
16-bit parameters must be the round-to-nearest-even of the masters."""
import pytest
import torch

import synth
from gpu_helpers import ADAMW_HP, TOL_ABS, TOL_REL
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("hp", [ADAMW_HP, (1e-2, 0.9, 0.999, 1e-8, 0.0), (3e-4, 0.9, 0.95, 1e-6, 0.1)])
def test_one_rank_step_follows_torch_adamw(hp):
    lr, b1, b2, eps, wd = hp
    P = 100_003
    w0 = synth.normal(P, 0.02, 4040, device="cuda")
    z = FlatZero(P, 1, "f32", "bf16")
    z.load_master(w0)
    p = torch.nn.Parameter(w0.clone())
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd, foreach=False)
    for k in range(1, 8):
        g = synth.normal(P, 1e-3, 4040 + k, device="cuda")
        z.grads[0].copy_(g)
        z.step(hp=hp)
        p.grad = g.clone()
        opt.step()
    torch.cuda.synchronize()
    st = opt.state[p]
    for mine, theirs, name in zip(z.current(), (p.detach(), st["exp_avg"], st["exp_avg_sq"]),
                                  ("master", "exp_avg", "exp_avg_sq")):
        err = (mine.double() - theirs.double()).abs()
        bound = TOL_REL * theirs.double().abs() + TOL_ABS
        bad = int((err > bound).sum())
        assert bad == 0, f"{name}: {bad} of {P} beyond tolerance, max error {float(err.max()):.3e}"
    assert torch.equal(z.params16.view(torch.int16), z.current()[0].to(torch.bfloat16).view(torch.int16))
    assert z.ctrl().step == 7
