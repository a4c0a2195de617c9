"""Host-side mixed-precision bit allocation from the sensitivity scores.

KronQ summary (hyper.ai), "Method" (Eq. 14): rank sublayers by
s = tr(H_G) tr(H_X) and give more bits to larger s; KronQ README (GitHub),
"Mapping paper results to flags": --inter_layer_mp upgrades the most
sensitive sublayers.

Rule for a 2/3/4-bit mix at a target average: every sublayer starts at
2 bits; the bit-parameters the target allows beyond that (a budget, an
integer) are handed out in descending score order, each sublayer taking the
widest width its parameters still fit into.  Equal scores keep the given
(decoder) order.  Among all allocations that keep the parameter-weighted
average at or below the target, this is the one with the most bits for the
most sensitive sublayer, then for the next, and so on.  Pure integer host
logic on the scores the GPU computed.
"""

from __future__ import annotations


def rank(scores) -> list:
    """Sublayer indices, most sensitive first; equal scores by index."""
    order = list(range(len(scores)))
    order.sort(key=lambda i: float(scores[i]), reverse=True)   # a stable sort keeps index order
    return order


def allocate_bits(scores, params, target_avg: float = 3.0, base: int = 2, top: int = 4) -> list:
    """Bits per sublayer (in the given order) from the scores and parameter counts."""
    counts = [int(p) for p in params]
    if len(counts) != len(scores):
        raise ValueError("one parameter count per score")
    if any(c <= 0 for c in counts):
        raise ValueError("parameter counts must be positive")
    total = sum(counts)
    spare = int(round(target_avg * total)) - base * total    # bit-params above the base width
    if spare < 0:
        raise ValueError("target average below the base width")
    out = [base] * len(counts)
    for i in rank(scores):
        extra = min(top - base, spare // counts[i])             # widest width that still fits
        out[i] = base + extra
        spare -= extra * counts[i]
    return out
