"""Workload shapes for weight-absorbed MLA decode.

Each workload is named for the model whose attention layer it is shaped like.
Shapes come from the pages' models:

* tiny: a 4-head, rank-32 layer used for parity at a size the oracle finishes
  instantly (contiguous cache).
* qwen25_7b: Qwen2.5-7B after MLAfication ("Why turn a GQA model into MLA" on
  the wzjinhao.cn page): 28 query heads in 4 KV groups, latent rank 128, 8 RoPE
  dims per KV group, so a cache row holds 128 + 4*8 = 160 numbers.
* deepseek_v2: DeepSeek-V2 attention ("Matrix absorption" section of the
  dtcms.com page): 128 heads, kv_lora_rank 512, qk_rope_head_dim 64 shared by
  all heads, qk_nope 128, v_head_dim 128.
* qwen3_30b_a3b: Qwen3-30B-A3B MLA delta (kwkr.cn page): 32 query heads in 4
  KV groups, rank 512, 8 RoPE dims per KV group, ragged context lengths.
* hybrid_*: the MLA layers of the zebra hybrid model (trdm.cn page):
  16 heads, kv_lora_rank 256, context extended to 1,048,576 tokens.
* prefill_*: one sequence's prefill chunk of q = 64, 256 or 1024 tokens attending
  causally over the cache (DeepSeek-V2 shape over 4,096 tokens; hybrid shape over 16,384).
* nanowhale_kv_shared: the single-latent K = V layer of nanowhale-100m (cnnetsun.cn
  page): 8 heads, one 512-d key/value vector per token with RoPE on its last 64 dims.

Model widths (``hidden_size``, the input of the KV down-projection): DeepSeek-V2 5120
(the dtcms.com page's o_proj is [128*128, 5120]), Qwen3-1.7B 2048 (trdm.cn page's
config table), nanowhale-100m 320 (cnnetsun.cn page). The pages print none for
Qwen2.5-7B or Qwen3-30B-A3B; reading: those models' published widths, 3584 and 2048.

This module holds shapes and seeds only; it does none of the method's
arithmetic.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class MLAConfig:
    name: str
    index: int                 # position in the workload list (seeds derive from it)
    batch: int                 # B
    q_len: int                 # q new query tokens per sequence
    num_heads: int             # H
    num_kv_groups: int         # G: groups sharing one rotated key slice (1 = shared k_pe)
    kv_lora_rank: int          # r
    qk_nope_dim: int           # d_n
    rope_dim: int              # d_r, RoPE dims per group
    v_head_dim: int            # d_v
    page_size: int = 64
    softmax_scale: float = 0.0
    context: int = 0           # fixed context length (when lens_range is None)
    lens_range: Optional[Tuple[int, int]] = None   # inclusive [lo, hi] for ragged lengths
    causal: bool = True        # causal inside the query block (matters when q_len > 1)
    contiguous: bool = False   # identity block table
    rope_base: float = 10000.0
    rope_ref_dim: int = 0      # denominator of the RoPE frequency exponent
    rope_index_pool: int = 0   # > 0: per-group frequency indices drawn from range(pool)
    with_bias: bool = False    # W_UV bias (the up_v.bias of the MLAfied checkpoints)
    identity_weights: bool = False   # W_UK = W_UV = I (needs d_n = d_v = r): plain MQA on c_kv
    hidden_size: int = 256     # model width feeding the KV down-projection (mla_down_kv_append)

    @property
    def row_width(self) -> int:
        """Numbers stored per cached token: latent plus every group's rotated key."""
        return self.kv_lora_rank + self.num_kv_groups * self.rope_dim

    @property
    def heads_per_group(self) -> int:
        return self.num_heads // self.num_kv_groups

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def with_(self, **kw) -> "MLAConfig":
        return replace(self, **kw)


def _cfg(**kw) -> MLAConfig:
    c = MLAConfig(**kw)
    if c.softmax_scale == 0.0:
        c = replace(c, softmax_scale=1.0 / math.sqrt(c.qk_nope_dim + c.rope_dim))
    if c.rope_ref_dim == 0:
        c = replace(c, rope_ref_dim=c.rope_dim)
    return c


TINY = _cfg(name="tiny", index=0, batch=1, q_len=1, num_heads=4, num_kv_groups=1,
            kv_lora_rank=32, qk_nope_dim=16, rope_dim=8, v_head_dim=16,
            context=256, contiguous=True, softmax_scale=1.0 / math.sqrt(24.0))

QWEN25_7B = _cfg(name="qwen25_7b", index=1, batch=32, q_len=1, num_heads=28,
                 num_kv_groups=4, kv_lora_rank=128, qk_nope_dim=128, rope_dim=8,
                 v_head_dim=128, context=4096, rope_ref_dim=128, rope_index_pool=64,
                 hidden_size=3584)

DEEPSEEK_V2 = _cfg(name="deepseek_v2", index=2, batch=64, q_len=1, num_heads=128,
                   num_kv_groups=1, kv_lora_rank=512, qk_nope_dim=128, rope_dim=64,
                   v_head_dim=128, context=8192, softmax_scale=1.0 / math.sqrt(192.0),
                   hidden_size=5120)

QWEN3_30B_A3B = _cfg(name="qwen3_30b_a3b", index=3, batch=128, q_len=1, num_heads=32,
                     num_kv_groups=4, kv_lora_rank=512, qk_nope_dim=128, rope_dim=8,
                     v_head_dim=128, lens_range=(1024, 32768), rope_ref_dim=128,
                     rope_index_pool=64, hidden_size=2048)

_HYB = dict(index=4, num_heads=16, num_kv_groups=1, kv_lora_rank=256, qk_nope_dim=128,
            rope_dim=64, v_head_dim=128, softmax_scale=1.0 / math.sqrt(192.0), hidden_size=2048)
HYBRID_1M_Q1 = _cfg(name="hybrid_1m_q1", batch=1, q_len=1, context=1 << 20, **_HYB)
HYBRID_1M_Q4 = _cfg(name="hybrid_1m_q4", batch=1, q_len=4, context=1 << 20, **_HYB)
HYBRID_256K_Q1 = _cfg(name="hybrid_256k_q1", batch=4, q_len=1, context=1 << 18, **_HYB)
HYBRID_256K_Q4 = _cfg(name="hybrid_256k_q4", batch=4, q_len=4, context=1 << 18, **_HYB)

# The single-latent K = V layer of nanowhale-100m (cnnetsun.cn page): 8 query heads over one
# KV head of head_dim 512 = 448 unrotated + 64 rotary dims, context 2,048. In the library's
# terms r = 448 and d_r = 64 with one key group; the output is the whole 512-d row.
NANOWHALE_KV_SHARED = _cfg(name="nanowhale_kv_shared", index=5, batch=128, q_len=1,
                           num_heads=8, num_kv_groups=1, kv_lora_rank=448, qk_nope_dim=448,
                           rope_dim=64, v_head_dim=512, context=2048,
                           softmax_scale=1.0 / math.sqrt(512.0), hidden_size=320)

# Prefill chunks: q new tokens attend causally over the latent cache they were appended to
# (the DeepSeek-V2 page's attention, with the query block of the hybrid workload's q = 4
# widened to a prefill chunk). One sequence, the DeepSeek-V2 and hybrid layer shapes.
PREFILL = {}
for _q in (64, 256, 1024):
    PREFILL[f"prefill_deepseek_v2_q{_q}"] = _cfg(
        name=f"prefill_deepseek_v2_q{_q}", index=6, batch=1, q_len=_q, num_heads=128,
        num_kv_groups=1, kv_lora_rank=512, qk_nope_dim=128, rope_dim=64, v_head_dim=128,
        context=4096, softmax_scale=1.0 / math.sqrt(192.0), hidden_size=5120)
    PREFILL[f"prefill_hybrid_q{_q}"] = _cfg(
        name=f"prefill_hybrid_q{_q}", index=7, batch=1, q_len=_q, num_heads=16,
        num_kv_groups=1, kv_lora_rank=256, qk_nope_dim=128, rope_dim=64, v_head_dim=128,
        context=16384, softmax_scale=1.0 / math.sqrt(192.0), hidden_size=2048)

CONFIGS = {c.name: c for c in (TINY, QWEN25_7B, DEEPSEEK_V2, QWEN3_30B_A3B, HYBRID_1M_Q1,
                               HYBRID_1M_Q4, HYBRID_256K_Q1, HYBRID_256K_Q4,
                               NANOWHALE_KV_SHARED, *PREFILL.values())}


def shrink(cfg: MLAConfig, batch: Optional[int] = None, context: Optional[int] = None,
           lens_range: Optional[Tuple[int, int]] = None, name: Optional[str] = None,
           **kw) -> MLAConfig:
    """Same head/rank geometry with fewer or shorter sequences (parity-size cases)."""
    upd = dict(kw)
    if batch is not None:
        upd["batch"] = batch
    if context is not None:
        upd["context"] = context
        upd["lens_range"] = None
    if lens_range is not None:
        upd["lens_range"] = lens_range
    upd["name"] = name or (cfg.name + "_small")
    return replace(cfg, **upd)
