"""Accounting of speculative verification blocks on the MoE layer.

"Understanding MoE Inference Costs on Galactus", section "Verification costs
belong to accepted output": a verification block runs the target model on the
candidate positions together, so the layer call reads the union of the
experts they select once, and what counts is that traffic per accepted token.
A block yields the target's own token plus the leading run of accepted drafted
tokens.  The layer call itself is the ordinary moe_layer_forward on the
block's positions; these helpers only count.
"""
from __future__ import annotations

from typing import Iterable


def accepted_tokens(accept_flags: Iterable[bool]) -> int:
    """Tokens one block outputs: 1 + the number of drafts accepted before the
    first rejection."""
    run = 0
    for ok in accept_flags:
        if not ok:
            break
        run += 1
    return run + 1


def expected_accepted_tokens(depth: int, alpha: float) -> float:
    """Mean tokens per block when each draft is accepted with probability alpha
    given that its predecessors were: 1 + alpha + ... + alpha^depth."""
    total, term = 0.0, 1.0
    for _ in range(depth + 1):
        total += term
        term *= alpha
    return total


def bytes_per_accepted_token(layer_bytes: float, accepted: float) -> float:
    """Layer traffic of the verification call divided by the tokens it accepted."""
    return layer_bytes / accepted
