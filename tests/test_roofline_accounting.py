"""Byte accounting of the roofline pinned to the sizes the pages print."""
import json
import os

from decoder_greedy_decode_b200 import roofline, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_byte_counts.json")


def test_lm_head_bytes_match_page():
    g = json.load(open(GOLDEN))
    mb = roofline.lm_head_bytes(synth.QWEN3_0_6B) / 1e6
    assert round(mb) == g["lm_head_bytes_per_token"]["value_mb"]


def test_mlp_bytes_match_page():
    g = json.load(open(GOLDEN))
    mb = roofline.mlp_bytes_per_token(synth.QWEN3_0_6B) / 1e6
    # the page prints 529 MB; gate+up+down of 28 layers are 528.48 MB
    assert abs(mb - g["mlp_bytes_per_token"]["value_mb"]) / g["mlp_bytes_per_token"]["value_mb"] < 0.002
    assert synth.QWEN3_0_6B.n_layers == g["n_layers"]["value"]


def test_step_bytes_0_6b_ctx_795():
    s = synth.QWEN3_0_6B
    assert roofline.layer_weight_params(s) == 15_730_944
    assert roofline.weight_bytes(s) == 1_192_099_840
    assert roofline.kv_bytes_per_token(s) == 114_688
    assert roofline.kv_bytes_per_token(s, "fp8") == 59_136
    assert roofline.step_bytes(s, [795]) == 1_192_099_840 + 796 * 114_688 + 2048


def test_step_bytes_1_7b():
    assert roofline.weight_bytes(synth.QWEN3_1_7B) == 3_441_149_952


def test_int8_weight_bytes_0_6b():
    """Weight-only int8: 28 x (15,728,640 projection codes + 12,288 row scales
    x 4 + 2,304 bf16 gains x 2) + lm_head (151,936 x 1,024 codes + 151,936 x 4)
    + the final norm (1,024 x 2)."""
    s = synth.QWEN3_0_6B
    assert roofline.projection_rows(s) == 12_288
    assert roofline.weight_bytes(s, "int8") == 28 * 15_782_400 + 156_190_208 + 2_048
    assert roofline.step_bytes(s, [795], weights="int8") == (
        598_099_456 + 796 * 114_688 + 2048)
