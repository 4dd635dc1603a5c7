"""Decode cost model T = C + S with S = B / W (test infrastructure only).

"Understanding MoE Inference Costs on Galactus", section "Turning throughput
into a cost estimate": the seconds per output token T split into a streaming
term S = B / W (B the expert bytes a token needs, W an effective bandwidth)
and a residual C = T - S that holds everything else.  The same arithmetic
turns the algorithmic bytes of one layer call into the time a bandwidth
ceiling allows (the roofline used when reporting measurements).
"""


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
