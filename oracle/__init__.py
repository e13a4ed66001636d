"""Float64 CPU oracle for the relation-KL loss and its gradient.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this package.  It shares no
code with the CUDA path (``attention_relation_kl_b200``), and the product path
never calls it.

``oracle.dense``  the definition (dense float64, optionally over row slabs).
``oracle.tiled``  tiled linear-memory restatements, checked against ``dense``.
``oracle.chain``  the chain rule to the student's projection weights.
``oracle.cast``   bfloat16 rounding (ties to even) of the float32 gradient.
"""
from . import cast, dense, tiled  # noqa: F401

__all__ = ["cast", "dense", "tiled"]
