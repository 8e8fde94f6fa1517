"""Which Linear layers of a Llama-3.x model take the FP8 path.

The FP8-Dynamic and FP8-Block checkpoints quantize every Linear layer except
the output head: lm_head sits on the ignore list and stays in high precision
("Llama-3.1-8B-Instruct-FP8-Dynamic" explainer, FP8 动态量化 table, lm_head
row; "Llama-3.1-70B-FP8-Dynamic" explainer, section 1.2; "Llama-3.2-3B-Instruct-
FP8-Block" explainer, quantization_config table, ignore).  The embedding is
not a Linear and never reaches this check.

Entries of an ignore list are module names matched exactly or as the last
dotted component(s) of a name ("lm_head" matches "lm_head" and
"model.lm_head"), or regular expressions written "re:<pattern>" matched
against the whole name.
"""
from __future__ import annotations

import re
from typing import Iterable

DEFAULT_IGNORE = ("lm_head",)


def _matches(name: str, entry: str) -> bool:
    if entry.startswith("re:"):
        return re.fullmatch(entry[3:], name) is not None
    return name == entry or name.endswith("." + entry)


def should_quantize(name: str, ignore: Iterable[str] = DEFAULT_IGNORE) -> bool:
    """True if the Linear layer `name` is stored and run in FP8."""
    return not any(_matches(name, e) for e in ignore)


def llama_linear_names(num_layers: int, tie_head: bool = False) -> list:
    """Module names of every Linear in a Llama-3.x decoder stack, in order."""
    names = []
    for i in range(num_layers):
        p = f"model.layers.{i}"
        names += [f"{p}.self_attn.q_proj", f"{p}.self_attn.k_proj", f"{p}.self_attn.v_proj",
                  f"{p}.self_attn.o_proj", f"{p}.mlp.gate_proj", f"{p}.mlp.up_proj",
                  f"{p}.mlp.down_proj"]
    if not tie_head:
        names.append("lm_head")
    return names


def kv_cache_bytes(context: int, layers: int, kv_heads: int, head_dim: int, element_bytes: float,
                   scale_bytes_per_head: int = 0) -> int:
    """Bytes of a K+V cache: context x layers x KV heads x head_dim x 2 (K and V)
    x bytes per element (the size model of the Llama-3.2-3B FP8-Block explainer,
    FAQ Q2), plus, for an FP8 cache with one scale per (token, head), that scale
    for each of K and V."""
    n = context * layers * kv_heads * 2
    return int(n * head_dim * element_bytes + n * scale_bytes_per_head)
