"""The five synthetic workloads, shaped like the LLaMA layers the KronQ pages
quantize (KronQ README (GitHub), "Model zoo"; KronQ summary (hyper.ai),
"Experiment": LLaMA-2-7B / LLaMA-3-8B / LLaMA-3-70B, 128 x 2048 calibration
tokens).

They stand in for WikiText-2 activations and real LLaMA weights, which are not
available here: X is heavy-tailed with a few outlier channels, G has
per-output-channel scales spread over several decades (the pages' Figure 1
shows diag(H_G) varying by orders of magnitude), W is Gaussian.
"""

from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class XSite:
    """One distinct layer input (several sublayers may read the same X)."""
    name: str
    width: int
    index: int


@dataclass(frozen=True)
class Sublayer:
    """One linear sublayer y = W x with W of shape m x n (m = d_out, n = d_in)."""
    name: str
    m: int
    n: int
    site: str
    index: int
    bits: int | None          # None: chosen by the mixed-precision allocation
    group: int                # -1 per-channel, else the group size along n


@dataclass(frozen=True)
class Config:
    name: str
    tokens: int
    sites: tuple
    sublayers: tuple
    w_std: float
    x_dist: str               # "normal" or "t4" (Student-t, 4 degrees of freedom)
    x_outlier_scale: float
    g_decades: float
    x_outliers_fixed: int | None = None   # fixed outlier count, else 0.5 % of the width
    w_row_logrange: tuple | None = None    # per-row std multiplier, log-uniform in this range
    w_round_bf16: bool = True
    alpha: float = 0.25
    damp: float = 0.01
    block: int = 128
    mode: str = "full"
    mixed_avg_bits: float | None = None
    seed: int = 0
    note: str = field(default="", compare=False)

    def site(self, name: str) -> XSite:
        for s in self.sites:
            if s.name == name:
                return s
        raise KeyError(name)

    def outlier_count(self, width: int) -> int:
        if self.x_outliers_fixed is not None:
            return self.x_outliers_fixed
        # 0.5 % of the channels, rounded half up
        return int((width * 5 + 500) // 1000)

    @property
    def weights(self) -> int:
        return sum(s.m * s.n for s in self.sublayers)


def _subs(specs, group, bits):
    return tuple(Sublayer(name=n, m=m, n=k, site=site, index=i, bits=bits, group=group)
                 for i, (n, m, k, site) in enumerate(specs))


TOY = Config(
    name="toy-256",
    tokens=2048,
    sites=(XSite("in", 256, 0),),
    sublayers=_subs([("linear", 256, 256, "in")], group=-1, bits=4),
    w_std=0.02, w_row_logrange=(0.5, 2.0), w_round_bf16=False,
    x_dist="normal", x_outliers_fixed=4, x_outlier_scale=20.0, g_decades=3.0,
    note="toy single linear layer, W4 asymmetric per-channel",
)

L2_7B_Q = Config(
    name="llama2-7b-q_proj",
    tokens=262144,
    sites=(XSite("attn_in", 4096, 0),),
    sublayers=_subs([("q_proj", 4096, 4096, "attn_in")], group=-1, bits=4),
    w_std=0.02, x_dist="t4", x_outlier_scale=20.0, g_decades=3.0,
    note="LLaMA-2-7B-shaped q_proj, W4 asymmetric per-channel",
)

L2_7B_MLP = Config(
    name="llama2-7b-mlp",
    tokens=262144,
    sites=(XSite("mlp_in", 4096, 0), XSite("down_in", 11008, 1)),
    sublayers=_subs([("gate_proj", 11008, 4096, "mlp_in"),
                     ("up_proj", 11008, 4096, "mlp_in"),
                     ("down_proj", 4096, 11008, "down_in")], group=128, bits=2),
    w_std=0.02, x_dist="t4", x_outlier_scale=20.0, g_decades=3.0,
    note="LLaMA-2-7B-shaped MLP, W2 asymmetric group-128",
)

L3_8B_BLOCK = Config(
    name="llama3-8b-block",
    tokens=262144,
    sites=(XSite("attn_in", 4096, 0), XSite("o_in", 4096, 1),
           XSite("mlp_in", 4096, 2), XSite("down_in", 14336, 3)),
    sublayers=_subs([("q_proj", 4096, 4096, "attn_in"),
                     ("k_proj", 1024, 4096, "attn_in"),
                     ("v_proj", 1024, 4096, "attn_in"),
                     ("o_proj", 4096, 4096, "o_in"),
                     ("gate_proj", 14336, 4096, "mlp_in"),
                     ("up_proj", 14336, 4096, "mlp_in"),
                     ("down_proj", 4096, 14336, "down_in")], group=-1, bits=None),
    w_std=0.02, x_dist="t4", x_outlier_scale=20.0, g_decades=3.0,
    mixed_avg_bits=3.0,
    note="LLaMA-3-8B-shaped decoder block, mixed 2/3/4-bit at a 3-bit average, per-channel",
)

L3_70B_MLP = Config(
    name="llama3-70b-mlp",
    tokens=262144,
    sites=(XSite("mlp_in", 8192, 0), XSite("down_in", 28672, 1)),
    sublayers=_subs([("gate_proj", 28672, 8192, "mlp_in"),
                     ("down_proj", 8192, 28672, "down_in")], group=128, bits=2),
    w_std=0.015, x_dist="t4", x_outlier_scale=30.0, g_decades=4.0,
    note="LLaMA-3-70B-shaped MLP, W2 asymmetric group-128",
)

CONFIGS = {c.name: c for c in (TOY, L2_7B_Q, L2_7B_MLP, L3_8B_BLOCK, L3_70B_MLP)}


def get_config(name: str) -> Config:
    return CONFIGS[name]
