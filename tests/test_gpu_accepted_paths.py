"""Decode paths the C ABI accepts beyond the benchmark shapes, each against the fp64 oracle
at the parity tolerances (2e-2 * max|ref| on o and o_latent, 1e-3 on lse):

* causal = 0 with several query rows (every row sees the whole context);
* rope_dim = 0, including the identity-weight case (W_UK = W_UV = I, d_n = d_v = r) in which
  the method reduces to multi-query attention over c_kv;
* more than 64 query rows on the one-CTA kernel, which runs them as 64-row blocks in
  lockstep (latent rank not a multiple of 128, or a rotary width the two-CTA kernel does
  not take), with one split and with the automatic plan.
"""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from mla_inputs.configs import MLAConfig, _cfg
from tests.gpu_harness import GpuProblem, check_sequence

pytestmark = pytest.mark.gpu


def _run(cfg: MLAConfig, num_splits: int = 0, spare: int = 2, q_scale: float = 1.0):
    prob = GpuProblem(make_workload(cfg, spare_pages=spare, q_scale=q_scale), num_splits=num_splits)
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(cfg.batch):
        check_sequence(prob, b, cfg.name)
    return prob


NON_CAUSAL = {
    # 32 heads x 4 rows = 128 rows: two 64-row blocks of the one-CTA kernel
    "qwen3_q4_noncausal": shrink(CONFIGS["qwen3_30b_a3b"], batch=3, lens_range=(70, 900),
                                 q_len=4, causal=False),
    # 16 heads x 4 rows on the hybrid shape (one 64-row block)
    "hybrid_q4_noncausal": shrink(CONFIGS["hybrid_1m_q4"], batch=2, context=1000, causal=False),
    # 128 heads x 2 rows: two 128-row blocks of the two-CTA kernel
    "deepseek_q2_noncausal": shrink(CONFIGS["deepseek_v2"], batch=2, context=333, q_len=2,
                                    causal=False),
}


@pytest.mark.parametrize("name", sorted(NON_CAUSAL))
def test_non_causal_query_block(name):
    _run(NON_CAUSAL[name])


def test_non_causal_differs_from_causal():
    """The two masks give different outputs for the earlier query rows (so the flag is seen)."""
    cfg = NON_CAUSAL["hybrid_q4_noncausal"]
    a = GpuProblem(make_workload(cfg))
    a.step()
    b = GpuProblem(make_workload(cfg.with_(causal=True)))
    b.step()
    torch.cuda.synchronize()
    assert not torch.equal(a.lse[:, 0], b.lse[:, 0])
    assert torch.equal(a.lse[:, -1], b.lse[:, -1]) or \
        float((a.lse[:, -1] - b.lse[:, -1]).abs().max()) <= 1e-6


ROPE0 = {
    # identity weights: multi-query attention over c_kv, 8 heads, rank 64
    "mqa_identity": _cfg(name="mqa_identity", index=20, batch=2, q_len=1, num_heads=8,
                         num_kv_groups=1, kv_lora_rank=64, qk_nope_dim=64, rope_dim=0,
                         v_head_dim=64, context=300, identity_weights=True),
    # identity weights with 4 causal query rows
    "mqa_identity_q4": _cfg(name="mqa_identity_q4", index=21, batch=2, q_len=4, num_heads=8,
                            num_kv_groups=1, kv_lora_rank=64, qk_nope_dim=64, rope_dim=0,
                            v_head_dim=64, context=131, identity_weights=True),
    # rope_dim = 0 with learned-shape weights and 128 heads (two 64-row blocks, rank 512)
    "rope0_128h": _cfg(name="rope0_128h", index=22, batch=2, q_len=1, num_heads=128,
                       num_kv_groups=1, kv_lora_rank=512, qk_nope_dim=128, rope_dim=0,
                       v_head_dim=128, context=200),
}


@pytest.mark.parametrize("name", sorted(ROPE0))
def test_rope_dim_zero(name):
    _run(ROPE0[name])


MANY_ROWS = {
    # rank 320 (not a multiple of 128): 128 heads run as two 64-row blocks
    "h128_r320": _cfg(name="h128_r320", index=23, batch=3, q_len=1, num_heads=128,
                      num_kv_groups=1, kv_lora_rank=320, qk_nope_dim=128, rope_dim=64,
                      v_head_dim=128, context=350, softmax_scale=1.0 / np.sqrt(192.0)),
    # rotary width G * d_r = 48: 96 heads as a 64-row and a ragged 32-row block
    "h96_g3_rope48": _cfg(name="h96_g3_rope48", index=24, batch=2, q_len=1, num_heads=96,
                          num_kv_groups=3, kv_lora_rank=256, qk_nope_dim=128, rope_dim=16,
                          v_head_dim=128, lens_range=(65, 700)),
}


@pytest.mark.parametrize("splits", [1, 0])
@pytest.mark.parametrize("name", sorted(MANY_ROWS))
def test_many_rows_on_one_cta_kernel(name, splits):
    _run(MANY_ROWS[name], num_splits=splits)


def test_many_rows_peaked_softmax():
    """The running-max moves on the row-block path (q scaled by 8)."""
    _run(MANY_ROWS["h128_r320"], num_splits=3, q_scale=8.0)
