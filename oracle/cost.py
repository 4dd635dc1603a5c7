"""Decode cost model T = C + S with S = B / W, and verification traffic per
accepted token (test infrastructure only).

"Understanding MoE Inference Costs on Galactus", section "Turning throughput
into a cost estimate": the seconds per output token T split into a streaming
term S = B / W (B the expert bytes a token needs, W an effective bandwidth)
and a residual C = T - S that holds everything else.  The same arithmetic
turns the algorithmic bytes of one layer call into the time a bandwidth
ceiling allows (the roofline used when reporting measurements).

Same page, section "Verification costs belong to accepted output": a
speculative verification block runs the target model on several candidate
positions at once; what matters is the traffic per *accepted* token.  The
block reads the union of the experts its positions select, and yields the
target's own token plus the accepted prefix of the drafted ones.
"""

import numpy as np


def streaming_time(bytes_needed: float, bandwidth: float) -> float:
    """S = B / W (seconds, for bytes and bytes/second)."""
    return bytes_needed / bandwidth


def token_time(residual: float, bytes_needed: float, bandwidth: float) -> float:
    """T = C + S."""
    return residual + streaming_time(bytes_needed, bandwidth)


def residual(token_seconds: float, streaming_seconds: float) -> float:
    """C = T - S."""
    return token_seconds - streaming_seconds


def tokens_per_second(token_seconds: float) -> float:
    return 1.0 / token_seconds


def expected_accepted(depth: int, alpha: float) -> float:
    """Expected output tokens of one verification block of `depth` drafted
    tokens when each is accepted with probability `alpha` given that every
    earlier one was (acceptance stops at the first rejection), plus the
    target model's own token: sum_{i=0..depth} alpha^i."""
    return float(sum(alpha ** i for i in range(depth + 1)))


def accepted_in_block(accept: np.ndarray) -> int:
    """Output tokens of one block from its per-draft accept flags: 1 plus the
    length of the leading run of accepted drafts."""
    n = 0
    for a in np.asarray(accept, dtype=bool):
        if not a:
            break
        n += 1
    return 1 + n


def expert_union(idx: np.ndarray) -> int:
    """Distinct experts a block's positions select (the weights it must read)."""
    return int(np.unique(np.asarray(idx).reshape(-1)).size)


def bytes_per_accepted_token(block_bytes: float, accepted_tokens: float) -> float:
    """Verification traffic per accepted token."""
    return block_bytes / accepted_tokens
