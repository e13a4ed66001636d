"""Seeded synthetic inputs for the chain rule from dX_s to the projection weights.

This module only *draws inputs* (and runs the model's own forward projections
that produce the relation inputs); it holds none of the relation-KL arithmetic
and none of its backward (no inverse rotation, no weight gradient).

What the inputs stand for.  In LinearARD only the student's Q/K/V projections
are trained (pith.science verdict page, ``minor_comments``; the abstract on the
mlsanity.com index page: the student is the RoPE-scaled copy of the frozen
teacher).  At one attention layer the teacher and the student start from the
same projection weights W_q, W_k, W_v; their hidden states differ because the
layers below already see different positions.  The stand-in:

* hidden states H_t ~ N(0, 1) of shape [B, N, D]; H_s = H_t + sigma * N(0, 1);
* shared weights W_x ~ N(0, 1/D) of shape [D, heads_x * d] (x in q, k, v);
* projections X = H W split into heads [B, heads, N, d]; Q and K then take
  rotate-half RoPE (the same rotation as ``workload.synthetic.rope_rotate``):
  the teacher at positions p = 0..N-1, the student at p / s; V takes none.

H_s and W are formed in float64 and rounded once (RNE) to bf16; the
projections of the rounded H and W run in float32 (these are inputs, and both
sides of every comparison consume the same rounded results), RoPE in float64,
and the projected Q/K/V are rounded once to bf16.  Draw order from one
``torch.Generator(seed)`` in float32 on the CPU: H_t, then the H_s noise, then
W_q, W_k, W_v.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import torch

from .synthetic import Workload, rope_rotate

__all__ = ["ChainWorkload", "CHAIN_CONFIGS", "generate_chain", "relation_workload"]


@dataclasses.dataclass(frozen=True)
class ChainWorkload:
    """Shapes and value recipe of one projection-gradient workload."""
    name: str
    B: int
    N: int
    D: int                 # model (hidden) dimension
    H: int                 # query heads
    H_kv: int              # key/value heads
    d: int                 # head dimension
    rope_base: float
    pi_factor: float       # student RoPE positions are p / pi_factor
    h_noise: float         # std of the student's hidden-state perturbation
    seed: int
    causal: bool = True

    def heads(self, rel: str) -> int:
        return self.H if rel == "q" else self.H_kv


# A small case the float64 oracle finishes in seconds, and the LLaMA2-7B layer
# shape (D = 4096, 32 heads of 128) at the 32K bench sequence length.
CHAIN_CONFIGS: Dict[str, ChainWorkload] = {
    "chain_small": ChainWorkload("chain_small", B=1, N=384, D=256, H=4, H_kv=2, d=64,
                                 rope_base=1e4, pi_factor=4.0, h_noise=0.1, seed=41),
    "chain_llama2_n32k": ChainWorkload("chain_llama2_n32k", B=1, N=32768, D=4096, H=32, H_kv=32,
                                       d=128, rope_base=1e4, pi_factor=8.0, h_noise=0.1, seed=42),
}


def _draw(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def generate_chain(cw: ChainWorkload) -> Dict[str, object]:
    """Draw the workload.  Returns, on the CPU, all bf16 and contiguous:

    ``h_t``, ``h_s``: [B, N, D]; ``w``: {rel: [D, heads * d]};
    ``x``: {rel: (x_teacher, x_student)} with x [B, heads, N, d] post-RoPE for
    q and k; ``pos_t``, ``pos_s``: the float64 RoPE positions [N].
    """
    gen = torch.Generator().manual_seed(cw.seed)
    ht = _draw(gen, (cw.B, cw.N, cw.D)).to(torch.float64)
    hs = ht + cw.h_noise * _draw(gen, (cw.B, cw.N, cw.D)).to(torch.float64)
    ht16, hs16 = ht.to(torch.bfloat16), hs.to(torch.bfloat16)
    w = {}
    for rel in ("q", "k", "v"):
        w[rel] = (_draw(gen, (cw.D, cw.heads(rel) * cw.d)).to(torch.float64)
                  / cw.D ** 0.5).to(torch.bfloat16)
    pos_t = torch.arange(cw.N, dtype=torch.float64)
    pos_s = pos_t / cw.pi_factor
    x = {}
    for rel in ("q", "k", "v"):
        hd = cw.heads(rel)
        wr = w[rel].to(torch.float32)
        pair = []
        for hx, pos in ((ht16, pos_t), (hs16, pos_s)):
            proj = (hx.to(torch.float32) @ wr).reshape(cw.B, cw.N, hd, cw.d).permute(0, 2, 1, 3)
            if rel != "v":
                proj = rope_rotate(proj, pos, cw.rope_base)
            pair.append(proj.to(torch.bfloat16).contiguous())
        x[rel] = tuple(pair)
    return {"h_t": ht16.contiguous(), "h_s": hs16.contiguous(),
            "w": {r: t.contiguous() for r, t in w.items()}, "x": x,
            "pos_t": pos_t, "pos_s": pos_s}


def relation_workload(cw: ChainWorkload) -> Workload:
    """The relation-KL workload (shapes, mask) that a chain workload feeds."""
    return Workload(cw.name, B=cw.B, H=cw.H, H_kv=cw.H_kv, N=cw.N, d=cw.d, dtype="bf16",
                    causal=cw.causal, relations=("q", "k", "v"), rope_base=cw.rope_base,
                    pi_factor=cw.pi_factor, v_noise=0.0, seed=cw.seed)
