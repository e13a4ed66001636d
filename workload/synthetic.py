"""Seeded synthetic teacher/student activations for the relation-KL path.

This module only *draws inputs*.  It holds none of the relation-KL arithmetic
(no logits, no softmax, no divergence, no gradient): both the float64 oracle
and the CUDA path consume exactly the tensors it returns.

What the inputs stand for.  LinearARD (arXiv 2604.00004, abstract; pith.science
verdict, ``pith_extraction.key_machinery``) distils the row-wise Q/Q, K/K and
V/V self-relation distributions of a frozen native-RoPE teacher into a
RoPE-scaled student.  The pages measure on real LLaMA2/LLaMA3/Mistral
activations, which are not available here, so seeded Gaussian activations of the
same head shapes stand in for them:

* Q and K: pre-RoPE vectors u ~ N(0, 1).  The teacher sees RoPE at the native
  positions p = 0..N-1; the student sees the *same* u rotated at p / s
  (positional interpolation by a factor s, "PI 4x" / "PI 8x" on the pages).
* V: V_t ~ N(0, 1); V_s = V_t + N(0, sigma^2) noise (V carries no RoPE).

RoPE follows RoFormer in the "rotate-half" pairing used by LLaMA: dimension i
is paired with i + d/2 and both rotate by the angle pos * base^(-2i/d).  Angles
and the rotation are evaluated in float64, then the result is rounded once
(round-to-nearest-even) to the configured dtype.

Draw order from one ``torch.Generator`` seeded with the config's seed, all in
float32 on the CPU: Q, then K, then V, then the V noise.  Shapes are
[B, H, N, d] (K and V use H_kv heads).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch

__all__ = ["Workload", "CONFIGS", "get_config", "sweep_config", "generate",
           "rope_rotate", "unit_list", "clustered_pair"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic relation-KL workload."""
    name: str
    B: int
    H: int                 # query heads (Q relation)
    H_kv: int              # key/value heads (K and V relations)
    N: int
    d: int
    dtype: str             # "bf16" or "fp32"
    causal: bool
    relations: Tuple[str, ...]   # subset of ("q", "k", "v"), in this order
    rope_base: float
    pi_factor: float       # student RoPE positions are p / pi_factor
    v_noise: float         # std of the student's V perturbation
    seed: int

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "fp32": torch.float32}[self.dtype]

    @property
    def gqa_group(self) -> int:
        return self.H // self.H_kv

    def heads(self, rel: str) -> int:
        return self.H if rel == "q" else self.H_kv

    @property
    def n_units(self) -> int:
        """Independent (batch, head, relation) problems."""
        return self.B * sum(self.heads(r) for r in self.relations)

    def causal_entries(self) -> int:
        """Valid (i, j) pairs of one unit's relation matrix."""
        return self.N * (self.N + 1) // 2 if self.causal else self.N * self.N


# The five workloads: a tiny single-head fp32 check, a LLaMA2-7B head block at
# 4K, the 32K extended-context training shape, a GQA LLaMA-3-8B block at 16K,
# and the sequence-length sweep (B * N = 65536).
CONFIGS: Dict[str, Workload] = {
    "tiny_fp32_n256": Workload("tiny_fp32_n256", B=1, H=1, H_kv=1, N=256, d=64,
                               dtype="fp32", causal=True, relations=("q",),
                               rope_base=1e4, pi_factor=4.0, v_noise=0.0, seed=1),
    "llama2_h32_n4k": Workload("llama2_h32_n4k", B=1, H=32, H_kv=32, N=4096, d=128,
                               dtype="bf16", causal=True, relations=("q", "k", "v"),
                               rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=2),
    "ext_h32_n32k": Workload("ext_h32_n32k", B=1, H=32, H_kv=32, N=32768, d=128,
                             dtype="bf16", causal=True, relations=("q", "k", "v"),
                             rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=3),
    "gqa_llama3_n16k": Workload("gqa_llama3_n16k", B=2, H=32, H_kv=8, N=16384, d=128,
                                dtype="bf16", causal=True, relations=("q", "k", "v"),
                                rope_base=5e5, pi_factor=4.0, v_noise=0.05, seed=4),
    # head dimension 64 (the smaller-head model class), otherwise the 32K shape
    "d64_h32_n32k": Workload("d64_h32_n32k", B=1, H=32, H_kv=32, N=32768, d=64,
                             dtype="bf16", causal=True, relations=("q", "k", "v"),
                             rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=6),
    # full (non-causal) mask: every row sees every token (the pages leave the
    # mask M open; this is the unmasked reading), 16K tokens
    "full_h32_n16k": Workload("full_h32_n16k", B=1, H=32, H_kv=32, N=16384, d=128,
                              dtype="bf16", causal=False, relations=("q", "k", "v"),
                              rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=7),
}

SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768, 65536)


def sweep_config(N: int) -> Workload:
    """One point of the sequence-length sweep: H=32, d=128, B = 65536 / N."""
    if N not in SWEEP_N:
        raise ValueError(f"sweep N must be one of {SWEEP_N}")
    return Workload(f"sweep_n{N}", B=65536 // N, H=32, H_kv=32, N=N, d=128,
                    dtype="bf16", causal=True, relations=("q", "k", "v"),
                    rope_base=1e4, pi_factor=8.0, v_noise=0.1, seed=5)


def get_config(name: str) -> Workload:
    if name in CONFIGS:
        return CONFIGS[name]
    if name.startswith("sweep_n"):
        return sweep_config(int(name[len("sweep_n"):]))
    raise KeyError(name)


def rope_rotate(u: torch.Tensor, positions: torch.Tensor, base: float) -> torch.Tensor:
    """Rotate-half RoPE of ``u`` [..., N, d] at float64 ``positions`` [N].

    Returns float64.  Dimension i pairs with i + d/2; both rotate by
    positions * base^(-2i/d) (RoFormer's rotary embedding).
    """
    d = u.shape[-1]
    if d % 2:
        raise ValueError("RoPE needs an even head dimension")
    half = d // 2
    inv_freq = base ** (-torch.arange(half, dtype=torch.float64) * 2.0 / d)
    ang = positions.to(torch.float64)[:, None] * inv_freq[None, :]          # [N, d/2]
    cos, sin = torch.cos(ang), torch.sin(ang)
    u64 = u.to(torch.float64)
    a, b = u64[..., :half], u64[..., half:]
    return torch.cat((a * cos - b * sin, b * cos + a * sin), dim=-1)


def _draw(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def generate(w: Workload) -> Dict[str, Tuple[torch.Tensor, torch.Tensor]]:
    """Draw the workload.  Returns {rel: (x_teacher, x_student)} on the CPU.

    Each tensor is contiguous [B, heads(rel), N, d] in ``w.torch_dtype``.
    """
    gen = torch.Generator().manual_seed(w.seed)
    pos_t = torch.arange(w.N, dtype=torch.float64)
    pos_s = pos_t / w.pi_factor
    out: Dict[str, Tuple[torch.Tensor, torch.Tensor]] = {}
    want = set(w.relations)
    # Draw order is fixed (Q, K, V, noise) whatever subset is requested, so a
    # relation's values do not depend on which others are asked for.
    q = _draw(gen, (w.B, w.H, w.N, w.d))
    k = _draw(gen, (w.B, w.H_kv, w.N, w.d)) if want & {"k", "v"} else None
    v = _draw(gen, (w.B, w.H_kv, w.N, w.d)) if "v" in want else None
    noise = _draw(gen, (w.B, w.H_kv, w.N, w.d)) if "v" in want else None
    dt = w.torch_dtype
    if "q" in want:
        out["q"] = (rope_rotate(q, pos_t, w.rope_base).to(dt).contiguous(),
                    rope_rotate(q, pos_s, w.rope_base).to(dt).contiguous())
    del q
    if "k" in want:
        out["k"] = (rope_rotate(k, pos_t, w.rope_base).to(dt).contiguous(),
                    rope_rotate(k, pos_s, w.rope_base).to(dt).contiguous())
    del k
    if "v" in want:
        vt = v.to(dt)
        vs = (v.to(torch.float64) + w.v_noise * noise.to(torch.float64)).to(dt)
        out["v"] = (vt.contiguous(), vs.contiguous())
    return {r: out[r] for r in w.relations}


def unit_list(w: Workload):
    """Unit order used by the fused Q/K/V launch: relation, then batch, then head."""
    return [(rel, b, h) for rel in w.relations for b in range(w.B) for h in range(w.heads(rel))]


def tiny_custom(N: int, d: int, dtype: str = "fp32", seed: int = 0, rope_base: float = 1e4,
                pi_factor: float = 4.0, causal: bool = True, B: int = 1, H: int = 1) -> Workload:
    """A small Q-relation workload of arbitrary shape for parity and edge cases."""
    return Workload(f"custom_b{B}h{H}n{N}d{d}{dtype}", B=B, H=H, H_kv=H, N=N, d=d, dtype=dtype,
                    causal=causal, relations=("q",), rope_base=rope_base,
                    pi_factor=pi_factor, v_noise=0.0, seed=seed)


def gaussian_pair(shape, seed: int, noise: float, dtype: torch.dtype = torch.float32):
    """x_t ~ N(0,1) and x_s = x_t + N(0, noise^2), drawn in that order."""
    gen = torch.Generator().manual_seed(seed)
    xt = _draw(gen, shape)
    xs = xt.to(torch.float64) + noise * _draw(gen, shape).to(torch.float64)
    return xt.to(dtype).contiguous(), xs.to(dtype).contiguous()


def clustered_pair(shape, seed: int, n_clusters: int = 4, amplitude: float = 2.5,
                   spread: float = 0.5, student_noise: float = 0.3,
                   dtype: torch.dtype = torch.bfloat16):
    """Rows drawn around a few shared directions, for logits far larger than
    unit-variance activations give.

    Draw order: cluster centres c ~ N(0,1) [n_clusters, d], the cluster of each
    row (uniform), the teacher's spread eps ~ N(0,1), the student's noise
    eta ~ N(0,1).  x_t = amplitude * c[k(row)] + spread * eps and
    x_s = x_t + student_noise * eta.  Rows of one cluster share a large common
    component, so with the 1/sqrt(d) scale their mutual logits sit near
    amplitude^2 sqrt(d) (about 70 for amplitude 2.5 and d = 128) rather than on
    the diagonal alone, and each row's distribution spreads over its cluster.
    """
    *lead, n, d = shape
    gen = torch.Generator().manual_seed(seed)
    centres = _draw(gen, (n_clusters, d)).to(torch.float64)
    which = torch.randint(0, n_clusters, tuple(lead) + (n,), generator=gen)
    eps = _draw(gen, shape).to(torch.float64)
    eta = _draw(gen, shape).to(torch.float64)
    xt = amplitude * centres[which] + spread * eps
    xs = xt + student_noise * eta
    return xt.to(dtype).contiguous(), xs.to(dtype).contiguous()
