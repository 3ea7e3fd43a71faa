"""Host-side dispatch policy for the fused op
("vllm_omni.diffusion.layers.fused_qk_norm_rope": fused_qk_norm_rope_min_tokens).

Each fused call pays a fixed host cost (argument checks, the launch), and
what it saves on the GPU scales with the number of tokens, so small calls may
do better with a consumer's unfused chain. The consumer passes the
crossover it measured on its own hardware as `default`; one environment
variable overrides it for every consumer of a deployment. The variable is read
at each call, so it can change without re-importing anything.
"""
from __future__ import annotations

import os
import re

ENV_MIN_TOKENS = "VLLM_OMNI_FUSED_QK_NORM_ROPE_MIN_TOKENS"
_INT = re.compile(r"[0-9]+")


def fused_qk_norm_rope_min_tokens(default: int) -> int:
    """The smallest token count for which a consumer should take the fused op.

    The environment variable, when set and not blank, must be a non-negative
    decimal integer (0 = always fuse); anything else raises ValueError. Unset
    or blank gives `default`.
    """
    raw = os.environ.get(ENV_MIN_TOKENS)
    if raw is None or raw.strip() == "":
        return int(default)
    text = raw.strip()
    if not _INT.fullmatch(text):
        raise ValueError(f"{ENV_MIN_TOKENS}={raw!r} is not a non-negative integer")
    return int(text)


def should_fuse(num_tokens: int, default: int) -> bool:
    """True when a call over num_tokens tokens should take the fused path."""
    return num_tokens >= fused_qk_norm_rope_min_tokens(default)
