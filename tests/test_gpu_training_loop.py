"""The library as the optimizer of a small model.

A two-layer MLP whose bf16 weights are views into the library's replicated
16-bit parameter buffer learns a fixed teacher network: every step, R = 2
data-parallel "ranks" each compute the gradient of their own micro-batch
(torch autograd on bf16 weights) into their gradient buffer, and one fused
call reduces, updates the fp32 masters and writes the new bf16 weights the
next forward pass reads.  The loss must fall well below its start, and a
twin run in which torch.optim.AdamW updates fp32 weights from the same
reduced gradients must reach about the same loss."""
import math

import pytest
import torch

from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu

D_IN, D_H, D_OUT, BATCH, R = 64, 256, 16, 512, 2
SHAPES = [(D_H, D_IN), (D_H,), (D_OUT, D_H), (D_OUT,)]
HP = (3e-3, 0.9, 0.999, 1e-8, 0.0)


def _forward(params, x):
    w1, b1, w2, b2 = params
    return torch.relu(x @ w1.t() + b1) @ w2.t() + b2


def _loss(params, x, y):
    return ((_forward(params, x).float() - y) ** 2).mean()


def _views(flat):
    out, off = [], 0
    for s in SHAPES:
        n = math.prod(s)
        out.append(flat[off:off + n].view(s))
        off += n
    return out


def test_two_rank_training_loop_learns_a_teacher():
    g = torch.Generator(device="cuda").manual_seed(7)
    P = sum(math.prod(s) for s in SHAPES)
    teacher = [torch.randn(s, device="cuda", generator=g) / math.sqrt(s[-1]) for s in SHAPES]
    w0 = torch.cat([(torch.randn(s, device="cuda", generator=g) / math.sqrt(s[-1])).flatten() for s in SHAPES])

    z = FlatZero(P, R, "bf16", "bf16")
    z.load_master(w0)
    weights16 = _views(z.params16)                     # the model's bf16 weights live in the library's buffer
    ref = torch.nn.Parameter(w0.clone())               # the twin: fp32 weights, torch AdamW
    opt = torch.optim.AdamW([ref], lr=HP[0], betas=HP[1:3], eps=HP[3], weight_decay=HP[4], foreach=False)

    losses, ref_losses = [], []
    for step in range(200):
        batches = []
        for r in range(R):
            x = torch.randn(BATCH, D_IN, device="cuda", generator=g)
            batches.append((x, _forward(teacher, x)))
        for r, (x, y) in enumerate(batches):
            params = [w.detach().requires_grad_(True) for w in weights16]
            loss = _loss(params, x.to(torch.bfloat16), y)
            grads = torch.autograd.grad(loss, params)
            torch.cat([gr.flatten() for gr in grads], out=z.grads[r])   # rank r's bf16 gradient
        losses.append(float(_loss(weights16, batches[0][0].to(torch.bfloat16), batches[0][1])))
        z.step(hp=HP)

        ref_grads = []
        for x, y in batches:
            params = [w.detach().requires_grad_(True) for w in _views(ref.detach())]
            grads = torch.autograd.grad(_loss(params, x, y), params)
            ref_grads.append(torch.cat([gr.flatten() for gr in grads]))
        ref_losses.append(float(_loss(_views(ref.detach()), batches[0][0], batches[0][1])))
        ref.grad = sum(ref_grads) / R                                   # the equal-weight mean
        opt.step()
    torch.cuda.synchronize()
    start, end = sum(losses[:5]) / 5, sum(losses[-5:]) / 5
    ref_end = sum(ref_losses[-5:]) / 5
    assert end < 0.1 * start, (start, end)
    assert end < 2.0 * ref_end + 1e-3, (end, ref_end)
    assert z.ctrl().step == 200
