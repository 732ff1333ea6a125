"""Layer shapes and input recipes of the five synthetic workloads.

Dimensions of the K3-shape layer (hidden 7168, latent 3584, 896 routed experts
with top-16, expert intermediate 3072, 2 shared experts) are the ones the
dimension table of "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか"
(section "K3のエキスパートは896個の小型LLMではない") lists.  The shared-expert
intermediate (3072) is not printed there and is an assumption.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int  # tokens
    H: int  # hidden
    L: int  # latent
    E: int  # routed experts
    k: int  # experts per token
    I: int  # routed-expert intermediate
    S: int  # shared experts
    Is: int  # shared-expert intermediate
    act: str = "bf16"  # activations / dense weights: "f32" or "bf16"
    # routed-expert weights: "f32", "bf16", "mxfp4", "mxfp4_a8" or "mxfp4_a4"
    # (MXFP4 weights with the experts' inputs quantised to MXFP8 / MXFP4: the
    # block-scaled paths)
    routed: str = "bf16"
    bias: str = "normal"  # "normal" (N(0, bias_std)) or "zipf"
    bias_std: float = 0.05
    zipf_s: float = 0.8
    gamma: str = "ones"  # "ones" or "normal" (1 + N(0, 0.1))
    seed: int = 0
    oracle_tokens: int | None = None  # tokens the oracle checks (None = all)
    situ_c: float = 10.0
    rms_eps: float = 1e-6

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)

    # --- algorithmic work (counts only the k selected experts per token) ---
    def flops_per_token(self) -> int:
        H, L, E, k, I, S, Is = self.H, self.L, self.E, self.k, self.I, self.S, self.Is
        router = 2 * H * E
        down = 2 * H * L
        experts = k * (2 * L * 2 * I + 2 * I * L)
        shared = S * (2 * H * 2 * Is + 2 * Is * H)
        up = 2 * L * H
        return router + down + experts + shared + up

    def expert_flops_per_token(self) -> tuple[int, int]:
        """(gate/up, down) flops per token over its k experts."""
        return self.k * 2 * self.L * 2 * self.I, self.k * 2 * self.I * self.L


CONFIGS: dict[str, LayerConfig] = {
    "tiny": LayerConfig("tiny", T=64, H=256, L=128, E=32, k=4, I=128, S=1, Is=256, act="f32", routed="f32"),
    "mid": LayerConfig("mid", T=4096, H=2048, L=1024, E=128, k=8, I=768, S=2, Is=1024),
    "decode": LayerConfig("decode", T=256, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072),
    "prefill": LayerConfig("prefill", T=16384, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072, bias="zipf",
                           oracle_tokens=512),
    "mxfp4": LayerConfig("mxfp4", T=8192, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072, routed="mxfp4",
                         oracle_tokens=512),
    # Small MXFP4 layer for parity tests (L and I multiples of 512 as the
    # block-scaled path requires).
    "mxfp4-small": LayerConfig("mxfp4-small", T=1024, H=2048, L=1024, E=64, k=8, I=1024, S=2, Is=1024,
                               routed="mxfp4"),
    # Profiling stand-in for the prefill layer: K3 matrix shapes, 64 experts
    # (4.2 GB of routed weights instead of 59 GB) so that multi-pass counter
    # captures stay small; not a measured workload.
    "prefill-e64": LayerConfig("prefill-e64", T=1024, H=7168, L=3584, E=64, k=16, I=3072, S=2, Is=3072, bias="zipf",
                               oracle_tokens=64),
    # The same stand-in with MXFP4 routed weights (1.1 GB of codes and scales).
    "mxfp4-e64": LayerConfig("mxfp4-e64", T=1024, H=7168, L=3584, E=64, k=16, I=3072, S=2, Is=3072, bias="zipf",
                             routed="mxfp4", oracle_tokens=64),
    # Block-scaled variant: MXFP4 routed weights x MXFP8 expert inputs, at the
    # MXFP4 workload's size, a small parity layer and a profiling stand-in.
    "mxfp4-a8": LayerConfig("mxfp4-a8", T=8192, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072,
                            routed="mxfp4_a8", oracle_tokens=512),
    "mxfp4a8-small": LayerConfig("mxfp4a8-small", T=1024, H=2048, L=1024, E=64, k=8, I=1024, S=2, Is=1024,
                                 routed="mxfp4_a8"),
    "mxfp4a8-e64": LayerConfig("mxfp4a8-e64", T=1024, H=7168, L=3584, E=64, k=16, I=3072, S=2, Is=3072, bias="zipf",
                               routed="mxfp4_a8", oracle_tokens=64),
    # All-4-bit variant: MXFP4 routed weights x MXFP4 expert inputs, the same
    # three sizes.
    "mxfp4-a4": LayerConfig("mxfp4-a4", T=8192, H=7168, L=3584, E=896, k=16, I=3072, S=2, Is=3072,
                            routed="mxfp4_a4", oracle_tokens=512),
    "mxfp4a4-small": LayerConfig("mxfp4a4-small", T=1024, H=2048, L=1024, E=64, k=8, I=1024, S=2, Is=1024,
                                 routed="mxfp4_a4"),
    "mxfp4a4-e64": LayerConfig("mxfp4a4-e64", T=1024, H=7168, L=3584, E=64, k=16, I=3072, S=2, Is=3072, bias="zipf",
                               routed="mxfp4_a4", oracle_tokens=64),
}

# Tensor ids: the second half of the Philox key of each input tensor.
TID = {
    "x": 1,
    "Wr": 2,
    "bias": 3,
    "Wdown": 4,
    "Wup": 5,
    "gamma": 6,
    "Wg": 7,
    "Wv": 8,
    "Wo": 9,
    "Wsg": 10,
    "Wsv": 11,
    "Wso": 12,
    "zipf_perm": 13,
    "sample": 14,
    "qb_scores": 15,
}


def tensor_shape(cfg: LayerConfig, name: str) -> tuple[int, ...]:
    H, L, E, I, S, Is, T = cfg.H, cfg.L, cfg.E, cfg.I, cfg.S, cfg.Is, cfg.T
    return {
        "x": (T, H),
        "Wr": (E, H),
        "bias": (E,),
        "Wdown": (L, H),
        "Wup": (H, L),
        "gamma": (L,),
        "Wg": (E, I, L),
        "Wv": (E, I, L),
        "Wo": (E, L, I),
        "Wsg": (S, Is, H),
        "Wsv": (S, Is, H),
        "Wso": (S, H, Is),
    }[name]


def tensor_std(cfg: LayerConfig, name: str) -> float:
    """Standard deviation of each tensor: x ~ N(0,1), weights ~ N(0, 1/fan_in)."""
    H, L, I, Is = cfg.H, cfg.L, cfg.I, cfg.Is
    return {
        "x": 1.0,
        "Wr": H ** -0.5,
        "bias": cfg.bias_std,
        "Wdown": H ** -0.5,
        "Wup": L ** -0.5,
        "gamma": 0.1,
        "Wg": L ** -0.5,
        "Wv": L ** -0.5,
        "Wo": I ** -0.5,
        "Wsg": H ** -0.5,
        "Wsv": H ** -0.5,
        "Wso": Is ** -0.5,
    }[name]


def tensor_dtype(cfg: LayerConfig, name: str) -> str:
    """Storage type of each input: 'f32', 'bf16' or 'mxfp4'."""
    if name in ("bias", "gamma"):
        return "f32"
    if name in ("Wg", "Wv", "Wo"):
        return "mxfp4" if cfg.routed in ("mxfp4_a8", "mxfp4_a4") else cfg.routed
    return cfg.act
