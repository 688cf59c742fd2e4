"""Prefill chunks (q = 64, 256, 1024 new tokens attending causally over the latent cache) on
the GPU against the fp64 oracle of the unabsorbed form: several blocks of 128 query rows per
sequence on the two-CTA kernel, read in lockstep, at context lengths the oracle finishes in
seconds (sampled heads for the 128-head shape), and at the benchmark sizes on sampled
query rows and heads."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import LSE_TOL, O_TOL, GpuProblem, max_rel_err

pytestmark = pytest.mark.gpu


def _check_heads(prob, b, heads, rows=None, what=""):
    ref = prob.oracle_heads(b, heads)
    rows = slice(None) if rows is None else rows
    got_o = prob.o[b][rows][:, heads].float().cpu().numpy()
    got_ol = prob.o_latent[b][rows][:, heads].float().cpu().numpy()
    got_lse = prob.lse[b][rows][:, heads].cpu().numpy()
    ref_o = np.stack([ref[h]["o"][rows] for h in heads], axis=1)
    ref_ol = np.stack([ref[h]["o_latent"][rows] for h in heads], axis=1)
    ref_lse = np.stack([ref[h]["lse"][rows] for h in heads], axis=1)
    assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_lse)), what
    assert max_rel_err(got_o, ref_o) <= O_TOL, f"{what}: o {max_rel_err(got_o, ref_o):.3e}"
    assert max_rel_err(got_ol, ref_ol) <= O_TOL, f"{what}: o_latent"
    assert float(np.max(np.abs(got_lse - ref_lse))) <= LSE_TOL, f"{what}: lse"


SMALL = {
    "deepseek_q64": shrink(CONFIGS["prefill_deepseek_v2_q64"], context=333),
    "deepseek_q256": shrink(CONFIGS["prefill_deepseek_v2_q256"], context=700, batch=2),
    "hybrid_q64": shrink(CONFIGS["prefill_hybrid_q64"], context=500, batch=2),
    "hybrid_q1024": shrink(CONFIGS["prefill_hybrid_q1024"], context=1500),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_prefill_parity(name):
    cfg = SMALL[name]
    prob = GpuProblem(make_workload(cfg, spare_pages=2))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    H = cfg.num_heads
    heads = list(range(H)) if H <= 16 else [0, 1, 63, 64, 127]
    for b in range(cfg.batch):
        _check_heads(prob, b, heads, what=f"{name} seq {b}")


def test_prefill_q1024_deepseek_sampled():
    """1024 query rows x 128 heads = 1024 row blocks of the two-CTA kernel."""
    cfg = shrink(CONFIGS["prefill_deepseek_v2_q1024"], context=1200)
    prob = GpuProblem(make_workload(cfg))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    _check_heads(prob, 0, [0, 77, 127], what="deepseek q1024")


@pytest.mark.parametrize("name", ["prefill_deepseek_v2_q256", "prefill_hybrid_q1024"])
def test_prefill_full_size_sampled(name):
    """The benchmark sizes, in the bench's launch configuration: first, middle and last query
    rows of sampled heads against the oracle; every row finite."""
    cfg = CONFIGS[name]
    prob = GpuProblem(make_workload(cfg))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    assert bool(torch.isfinite(prob.o.float()).all()) and bool(torch.isfinite(prob.lse).all())
    q = cfg.q_len
    rows = np.array([0, q // 2, q - 1])
    heads = [0, cfg.num_heads - 1]
    _check_heads(prob, 0, heads, rows=rows, what=name)
