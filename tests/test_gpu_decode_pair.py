"""Decode with more than 64 query rows per sequence: blocks of 128 rows on clusters of two
CTAs that split the latent; each CTA runs the softmax of half the rows on its own and the
partner's partial scores (swapped through distributed shared memory) and returns the
weights. Parity with the fp64 oracle of the unabsorbed form on the shapes that take this
path: several row blocks, padding rows past q*H, ranks 256 / 384 / 512, rotary widths 32 /
64 / 128 (the three shared-memory swizzles of Q's rotary half), ragged and edge lengths;
plus split and paging invariance and the bounds guard on this path."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import GpuProblem, check_sequence

pytestmark = pytest.mark.gpu

DS = CONFIGS["deepseek_v2"]
HYB = CONFIGS["hybrid_1m_q1"]

PAIR = {
    # 128 heads, q = 2: two row blocks of 128, causal inside the query block
    "deepseek_q2": shrink(DS, batch=2, context=450, q_len=2),
    # 96 heads: one block with 32 padding rows
    "heads96": shrink(DS, batch=2, context=333, num_heads=96, name="heads96"),
    # rank 256, 16 heads x 8 query tokens = 128 rows (rotary half 32)
    "rank256_q8": shrink(HYB, batch=2, context=700, q_len=8, name="rank256_q8"),
    # ragged lengths, many sequences: pieces cut between clusters are merged
    "deepseek_ragged": shrink(DS, batch=9, lens_range=(1, 900), name="deepseek_ragged"),
    # heads sharing 4 rotary groups of 16: rotary half 32
    "groups4": shrink(DS, batch=2, context=260, num_kv_groups=4, rope_dim=16, name="groups4"),
    # rank 384: three latent blocks per CTA, one of them from shared memory
    "rank384": shrink(DS, batch=2, context=300, kv_lora_rank=384, name="rank384"),
    # 2 groups x 64 rotary dims: rotary half 64 (128-byte swizzle), fewer cache slots
    "rope128": shrink(DS, batch=2, context=400, num_kv_groups=2, rope_dim=64, name="rope128"),
    # 32 rotary dims shared by all heads: rotary half 16 (32-byte swizzle, one K step)
    "rope32": shrink(DS, batch=2, context=350, rope_dim=32, name="rope32"),
    # 32 heads x 4 query tokens: causal inside the block, 128 rows
    "heads32_q4": shrink(HYB, batch=3, context=500, num_heads=32, q_len=4, kv_lora_rank=512,
                         name="heads32_q4"),
}


@pytest.mark.parametrize("name", sorted(PAIR))
def test_pair_decode_parity(name):
    cfg = PAIR[name]
    assert cfg.q_len * cfg.num_heads > 64
    prob = GpuProblem(make_workload(cfg, spare_pages=2))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(cfg.batch):
        check_sequence(prob, b, name)


@pytest.mark.parametrize("lens", [[1], [64], [65], [2, 128, 129, 63]])
def test_pair_edge_lengths(lens):
    cfg = shrink(DS, batch=len(lens), context=max(lens), name="pair_edge")
    prob = GpuProblem(make_workload(cfg, seq_lens=np.array(lens, dtype=np.int32)))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(len(lens)):
        check_sequence(prob, b, f"lens={lens}")


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_pair_split_count(splits):
    """Every split count gives the oracle's answer (0 = one range per resident cluster)."""
    cfg = PAIR["deepseek_ragged"]
    prob = GpuProblem(make_workload(cfg), num_splits=splits)
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in (0, 4, 8):
        check_sequence(prob, b, f"splits={splits}")


def test_pair_paging_invariance_and_determinism():
    cfg = PAIR["deepseek_ragged"]
    wl = make_workload(cfg, spare_pages=7)
    a = GpuProblem(wl, num_splits=2)
    a.step()
    perm = np.random.default_rng(5).permutation(wl.num_pages)
    table2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    b = GpuProblem(wl, num_splits=2, block_table=table2)
    b.step()
    torch.cuda.synchronize()
    assert torch.equal(a.o_latent, b.o_latent)
    assert torch.equal(a.lse, b.lse)
    o_prev = a.o_latent.clone()
    a.decode_only(num_splits=2)
    torch.cuda.synchronize()
    assert torch.equal(a.o_latent, o_prev), "repeated decode is not bitwise identical"


def test_pair_bad_page_id_is_flagged_not_faulted():
    cfg = shrink(DS, batch=3, context=300, name="pair_bad_page")
    wl = make_workload(cfg)
    prob = GpuProblem(wl, num_splits=1)
    prob.step()
    torch.cuda.synchronize()
    bad = wl.block_table.copy()
    bad[1, 2] = wl.num_pages + 1000
    prob.block_table = torch.from_numpy(bad).cuda()
    prob.decode_only()
    assert mla.mla_get_device_status(prob.workspace.view(torch.int32)[:1], reset=True) == \
        mla.MLA_ERR_DEVICE_BOUNDS
    check_sequence(prob, 0, "bad page, seq 0")
    check_sequence(prob, 2, "bad page, seq 2")
