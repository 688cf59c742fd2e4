"""Decode parity at the full benchmark sizes, in the launch configuration the bench times
(automatic split plan, same calls), on sampled outputs the fp64 oracle computes one head at
a time, plus properties every output row must have.

The oracle is the unabsorbed form; at these sizes it runs on a few (sequence, head) pairs
per config: the first and last sequence (and, with ragged lengths, the longest and the
shortest), and heads from the first, a middle and the last key group.
"""
import numpy as np
import pytest
import torch

from mla_inputs import CONFIGS, make_workload
from tests.gpu_harness import LSE_TOL, O_TOL, GpuProblem, max_rel_err

pytestmark = pytest.mark.gpu

FULL = ["qwen25_7b", "deepseek_v2", "qwen3_30b_a3b", "hybrid_1m_q1", "hybrid_1m_q4",
        "hybrid_256k_q1", "hybrid_256k_q4"]


def _sampled_sequences(lens: np.ndarray) -> list:
    picks = [0, len(lens) - 1, int(np.argmax(lens)), int(np.argmin(lens))]
    return sorted(set(picks))


def _sampled_heads(H: int, G: int, long_context: bool) -> list:
    per = H // G
    heads = [0, (G // 2) * per + per // 2, H - 1]
    # a head costs ~2 * L * r * (d_n + d_v) oracle FLOPs: one head per million-token sequence
    return [heads[1]] if long_context else sorted(set(heads))


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_parity(name):
    cfg = CONFIGS[name]
    wl = make_workload(cfg)
    prob = GpuProblem(wl)                      # num_splits = 0: the plan the bench times
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == 0

    # every row: finite, and o_latent a convex combination of cached latent rows
    o = prob.o.float()
    ol = prob.o_latent.float()
    lse = prob.lse
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(ol).all())
    assert bool(torch.isfinite(lse).all())
    bound = 0.0
    for b in range(cfg.batch):
        pages = prob.block_table[b, :(int(wl.seq_lens[b]) + cfg.page_size - 1) // cfg.page_size]
        rows = prob.cache[pages.long()].reshape(-1, cfg.row_width)[:int(wl.seq_lens[b]),
                                                                     :cfg.kv_lora_rank]
        bound = max(bound, float(rows.float().abs().max()))
    assert float(ol.abs().max()) <= bound * (1 + 2 ** -7)

    long_context = int(wl.seq_lens.max()) > 300_000
    heads = _sampled_heads(cfg.num_heads, cfg.num_kv_groups, long_context)
    seqs = _sampled_sequences(wl.seq_lens)
    if long_context:
        seqs = seqs[:2]
    for b in seqs:
        ref = prob.oracle_heads(b, heads)
        got_o = prob.o[b][:, heads].float().cpu().numpy()
        got_ol = prob.o_latent[b][:, heads].float().cpu().numpy()
        got_lse = prob.lse[b][:, heads].cpu().numpy()
        ref_o = np.stack([ref[h]["o"] for h in heads], axis=1)
        ref_ol = np.stack([ref[h]["o_latent"] for h in heads], axis=1)
        ref_lse = np.stack([ref[h]["lse"] for h in heads], axis=1)
        e_o, e_ol = max_rel_err(got_o, ref_o), max_rel_err(got_ol, ref_ol)
        e_lse = float(np.max(np.abs(got_lse - ref_lse)))
        what = f"{name} seq {b} (L={int(wl.seq_lens[b])}) heads {heads}"
        assert e_o <= O_TOL, f"{what}: o rel err {e_o:.3e}"
        assert e_ol <= O_TOL, f"{what}: o_latent rel err {e_ol:.3e}"
        assert e_lse <= LSE_TOL, f"{what}: lse err {e_lse:.3e}"
