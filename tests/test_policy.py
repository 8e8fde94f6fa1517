"""The ignore list (lm_head stays high precision) and the checkpoint facts
the pages print for the 70B FP8-Dynamic model, which pin what is quantized and
at what granularity: 560 weight_scale tensors, 70.56B parameters, 72.67 GB."""
import json
import os

import pytest

from fp8_w8a8_quantized_amax_b200 import policy

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def test_lm_head_is_not_quantized():
    assert FACTS["ignore_list"]["value"] == list(policy.DEFAULT_IGNORE)
    assert not policy.should_quantize("lm_head")
    assert not policy.should_quantize("model.lm_head")
    for n in ("model.layers.0.self_attn.q_proj", "model.layers.79.mlp.down_proj",
              "model.layers.3.mlp.gate_proj"):
        assert policy.should_quantize(n)


def test_regex_and_suffix_entries():
    ign = ("lm_head", "re:.*\\.mlp\\.gate_proj", "q_proj")
    assert not policy.should_quantize("model.layers.1.mlp.gate_proj", ign)
    assert not policy.should_quantize("model.layers.1.self_attn.q_proj", ign)
    assert policy.should_quantize("model.layers.1.mlp.up_proj", ign)
    assert policy.should_quantize("model.layers.1.self_attn.xq_proj", ign)


@pytest.mark.parametrize("arch,want", [("llama70b_arch", 560), ("llama8b_arch", 224), ("llama3b_arch", 196)])
def test_quantized_linear_counts(arch, want):
    names = policy.llama_linear_names(FACTS[arch]["layers"])
    assert sum(policy.should_quantize(n) for n in names) == want
    if arch == "llama70b_arch":
        assert want == FACTS["llama70b_weight_scale_tensors"]["value"]


def _llama70b_bytes(scale_bytes, quantize_head=False):
    a = FACTS["llama70b_arch"]
    h, f, v, L = a["hidden"], a["intermediate"], a["vocab"], a["layers"]
    kv = a["kv_heads"] * a["head_dim"]
    outs = {"q_proj": h, "k_proj": kv, "v_proj": kv, "o_proj": h,
            "gate_proj": f, "up_proj": f, "down_proj": h}
    ins = {"q_proj": h, "k_proj": h, "v_proj": h, "o_proj": h,
           "gate_proj": h, "up_proj": h, "down_proj": f}
    fp8_params = scales = 0
    for n in policy.llama_linear_names(L):
        if not policy.should_quantize(n):
            continue
        short = n.rsplit(".", 1)[1]
        fp8_params += outs[short] * ins[short]
        scales += outs[short]          # one scale per output channel
    bf16_params = 2 * v * h + (2 * L + 1) * h   # embedding, lm_head, RMSNorm weights
    if quantize_head:
        fp8_params += v * h
        scales += v
        bf16_params -= v * h
    params = fp8_params + scales + bf16_params
    return params, fp8_params + scales * scale_bytes + 2 * bf16_params


def test_llama70b_checkpoint_size_matches_page():
    params, nbytes = _llama70b_bytes(scale_bytes=2)
    assert round(params / 1e9, 2) == FACTS["llama70b_params_billion"]["value"]
    assert round(nbytes / 1e9, 2) == FACTS["llama70b_checkpoint_gb"]["value"]


def test_other_readings_do_not_match_the_page():
    # fp32 scales or an FP8 lm_head would not give the 72.67 GB the page prints
    assert round(_llama70b_bytes(scale_bytes=4)[1] / 1e9, 2) != 72.67
    assert round(_llama70b_bytes(scale_bytes=2, quantize_head=True)[1] / 1e9, 2) != 72.67


def test_kv_cache_size_model():
    # Llama-3.2-3B at its 128K context: 28 layers, 8 KV heads of 128 (FP8-Block explainer, FAQ Q2)
    from fp8_w8a8_quantized_amax_b200.policy import kv_cache_bytes
    bf16 = kv_cache_bytes(131072, 28, 8, 128, 2)
    assert bf16 == 131072 * 28 * 8 * 128 * 2 * 2 == 15032385536            # 15.0 GB
    fp8 = kv_cache_bytes(131072, 28, 8, 128, 1, scale_bytes_per_head=4)
    assert fp8 == bf16 // 2 + 131072 * 28 * 8 * 2 * 4                       # half, plus fp32 scales
    assert abs(fp8 / bf16 - (0.5 + 4 / (128 * 2))) < 1e-12                 # 1.6% of the bf16 size in scales
