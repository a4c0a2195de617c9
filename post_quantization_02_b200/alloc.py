"""Host-side mixed-precision bit allocation from the sensitivity scores.

KronQ summary (hyper.ai), "Method" (Eq. 14): rank sublayers by
s = tr(H_G) tr(H_X) and give more bits to larger s; KronQ README (GitHub),
"Mapping paper results to flags": --inter_layer_mp upgrades the most
sensitive sublayers by +1 bit.

For a 2/3/4-bit mix at a target average: every sublayer starts at 2 bits; in
descending score order each receives the largest upgrade (+2, else +1) that
keeps the parameter-weighted average at or below the target.  Ties keep the
given (decoder) order.  Pure integer host logic on the scores the GPU
computed.
"""

from __future__ import annotations


def rank(scores) -> list:
    scores = [float(s) for s in scores]
    return sorted(range(len(scores)), key=lambda i: (-scores[i], i))


def allocate_bits(scores, params, target_avg: float = 3.0, base: int = 2, top: int = 4) -> list:
    params = [int(p) for p in params]
    total = sum(params)
    budget = int(round(target_avg * total))
    bits = [base] * len(params)
    used = base * total
    for i in rank(scores):
        for up in range(top - base, 0, -1):
            if used + up * params[i] <= budget:
                bits[i] += up
                used += up * params[i]
                break
    return bits
