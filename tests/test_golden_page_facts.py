"""Workload shapes against the numbers the pages print (tests/golden/page_facts.json)."""
import json
import math
import os

from mla_inputs import CONFIGS

HERE = os.path.dirname(os.path.abspath(__file__))
FACTS = json.load(open(os.path.join(HERE, "golden", "page_facts.json")))


def test_qwen25_row_width_and_compression():
    c = CONFIGS["qwen25_7b"]
    gqa = FACTS["gqa_numbers_per_token_qwen25_7b"]
    assert math.prod(gqa["factors"]) == gqa["value"]
    mla = FACTS["mla_numbers_per_token_qwen25_7b"]
    assert c.row_width == mla["value"] == sum(mla["parts"])
    assert c.kv_lora_rank == mla["parts"][0]
    assert c.num_kv_groups * c.rope_dim == mla["parts"][1]
    assert gqa["value"] / c.row_width >= FACTS["compression_at_least"]["value"]


def test_deepseek_v2_shapes():
    c = CONFIGS["deepseek_v2"]
    q = FACTS["deepseek_v2_q_b_proj_out"]
    assert c.num_heads * (c.qk_nope_dim + c.rope_dim) == q["value"] == math.prod(q["factors"])
    assert [c.qk_nope_dim, c.rope_dim] == FACTS["deepseek_v2_q_head_split"]["value"]
    assert c.num_heads * c.v_head_dim == FACTS["deepseek_v2_o_proj_in"]["value"]
    assert [c.kv_lora_rank, c.row_width - c.kv_lora_rank] == FACTS["deepseek_v2_cache_row_split"]["value"]
    assert abs(c.softmax_scale - 1 / math.sqrt(c.qk_nope_dim + c.rope_dim)) < 1e-15
