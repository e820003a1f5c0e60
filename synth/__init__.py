"""Seeded synthetic inputs for the ZeRO-2/3 Adam step.

Shared by the tests and the benchmark, and by nothing else.  This module holds
shapes, seeds and random draws only -- none of the step's arithmetic.  Every
draw is reproducible from (base seed, workload id, kind, rank, step).

Workloads (all inputs synthetic; no dataset or checkpoint is involved):
  * "pages"     P=11, R=4: the worked example of "Deep dive: DeepSpeed",
                "Reduce first, then update the owned slice": w_i = 0.1*i,
                rank gradients ((i + 2r + step) mod 7 - 3) / 10.
  * "flat16m"   P=16,777,259 flat, R=8, bf16 gradients ~N(0, 1e-3).
  * "gpt2m"     GPT-2-medium tensor list (292 tensors, 354,823,168 params),
                R=4, fp16 gradients ~N(0, 1e-3) times a loss scale of 2^16.
  * "flat1p5b"  P=1.5e9 flat, R=4, bf16 (or fp32) gradients, token counts
                uniform in [1, 4096] per rank and step.
  * "llama3b"   Llama-style 3.2B tensor list (254 tensors), R=8, bf16.
Masters start ~N(0, 0.02); both moments start at zero.
"""
from __future__ import annotations

from typing import List, Tuple

import torch

BASE_SEED = 20261202

KIND_MASTER = 1
KIND_GRAD = 2
KIND_TOKENS = 3
KIND_INF = 4
KIND_SAMPLE = 5

_M64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _M64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _M64
    return x ^ (x >> 31)


def seed_for(workload: int, kind: int, rank: int = 0, step: int = 0) -> int:
    """A 63-bit seed for one independent stream of draws."""
    h = BASE_SEED
    for part in (workload, kind, rank, step):
        h = _splitmix64(h ^ (part & _M64))
    return h & ((1 << 63) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(n: int, std: float, seed: int, device="cpu", dtype=torch.float32,
           scale: float = 1.0) -> torch.Tensor:
    """n draws of N(0, std^2) (times `scale`), rounded once to `dtype`."""
    x = torch.randn(n, generator=_gen(seed, device), device=device, dtype=torch.float32)
    x.mul_(std * scale)
    return x.to(dtype)


def fill_normal_(out: torch.Tensor, std: float, seed: int, scale: float = 1.0) -> torch.Tensor:
    """Fill an existing tensor in place with N(0, std^2) draws (times `scale`)."""
    g = _gen(seed, out.device)
    if out.dtype == torch.float32:
        out.normal_(0.0, std * scale, generator=g)
        return out
    chunk = 1 << 26
    flat = out.view(-1)
    tmp = torch.empty(min(chunk, flat.numel()), device=out.device, dtype=torch.float32)
    for s in range(0, flat.numel(), chunk):
        e = min(s + chunk, flat.numel())
        t = tmp[: e - s]
        t.normal_(0.0, std * scale, generator=g)
        flat[s:e].copy_(t)
    return out


def pages_grads(P: int, R: int, step: int, dtype=torch.float32) -> List[torch.Tensor]:
    """The worked example's rank gradients ((i + 2r + step) mod 7 - 3) / 10."""
    i = torch.arange(P, dtype=torch.int64)
    return [(((i + 2 * r + step) % 7 - 3).to(torch.float64) / 10).to(dtype) for r in range(R)]


def pages_master(P: int, dtype=torch.float64) -> torch.Tensor:
    """The worked example's initial weights w_i = 0.1 * i."""
    return (torch.arange(P, dtype=torch.float64) * 0.1).to(dtype)


def token_counts(R: int, workload: int, step: int) -> List[int]:
    """Per-rank token counts, uniform integers in [1, 4096]."""
    g = _gen(seed_for(workload, KIND_TOKENS, 0, step), "cpu")
    return [int(x) for x in torch.randint(1, 4097, (R,), generator=g)]


def inf_site(workload: int, step: int, R: int, P: int) -> Tuple[int, int]:
    """(rank, index) where the overflow test plants an inf at this step."""
    h = seed_for(workload, KIND_INF, 0, step)
    return step % R, h % P


def sample_indices(P: int, n_random: int, workload: int, extra=()) -> torch.Tensor:
    """Sorted unique indices: both ends, `extra` positions and n random ones."""
    g = _gen(seed_for(workload, KIND_SAMPLE), "cpu")
    fixed = [0, 1, 2, 3, 4, 5, 6, 7, 8, P - 9, P - 8, P - 7, P - 3, P - 2, P - 1]
    idx = torch.cat([
        torch.tensor([x for x in list(fixed) + list(extra) if 0 <= x < P], dtype=torch.int64),
        torch.randint(0, P, (n_random,), generator=g, dtype=torch.int64)])
    return torch.unique(idx)


# ------------------------------------------------------------ tensor lists

def gpt2_medium_tensors() -> List[Tuple[str, int]]:
    """GPT-2 medium (24 layers, d=1024, FFN 4096, vocab 50257, tied embedding):
    292 parameter tensors in the usual named-parameter order."""
    d, ff, vocab, ctx, layers = 1024, 4096, 50257, 1024, 24
    out = [("wte", vocab * d), ("wpe", ctx * d)]
    for l in range(layers):
        p = f"h{l}."
        out += [(p + "ln_1.w", d), (p + "ln_1.b", d),
                (p + "attn.c_attn.w", d * 3 * d), (p + "attn.c_attn.b", 3 * d),
                (p + "attn.c_proj.w", d * d), (p + "attn.c_proj.b", d),
                (p + "ln_2.w", d), (p + "ln_2.b", d),
                (p + "mlp.c_fc.w", d * ff), (p + "mlp.c_fc.b", ff),
                (p + "mlp.c_proj.w", ff * d), (p + "mlp.c_proj.b", d)]
    out += [("ln_f.w", d), ("ln_f.b", d)]
    return out


def llama_3b_tensors() -> List[Tuple[str, int]]:
    """Llama-style 3.2B (28 layers, d=3072, FFN 8192, vocab 128256, 24 query
    and 8 KV heads of 128, tied embedding): 254 parameter tensors."""
    d, ff, vocab, layers, kv = 3072, 8192, 128256, 28, 8 * 128
    out = [("embed", vocab * d)]
    for l in range(layers):
        p = f"l{l}."
        out += [(p + "q", d * d), (p + "k", kv * d), (p + "v", kv * d), (p + "o", d * d),
                (p + "gate", ff * d), (p + "up", ff * d), (p + "down", d * ff),
                (p + "in_norm", d), (p + "post_norm", d)]
    out += [("norm", d)]
    return out


WORKLOADS = {
    "pages": 1,
    "flat16m": 2,
    "gpt2m": 3,
    "flat1p5b": 4,
    "llama3b": 5,
}

FLAT16M_P = 16_777_259
FLAT1P5B_P = 1_500_000_000
