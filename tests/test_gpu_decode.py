"""The full decode step (append -> absorb -> decode -> out_up) on the GPU against the
fp64 oracle of the unabsorbed form, at sizes the oracle finishes in seconds that still
span several pages and a ragged last page; plus split / paging invariance and the
device-side bounds guard."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import GpuProblem, check_sequence

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": CONFIGS["tiny"],
    "qwen25_7b": shrink(CONFIGS["qwen25_7b"], batch=3, context=777),
    "deepseek_v2": shrink(CONFIGS["deepseek_v2"], batch=2, context=517),
    "qwen3_30b_a3b": shrink(CONFIGS["qwen3_30b_a3b"], batch=4, lens_range=(60, 1500)),
    "hybrid_q1": shrink(CONFIGS["hybrid_1m_q1"], batch=2, context=3001),
    "hybrid_q4": shrink(CONFIGS["hybrid_1m_q4"], batch=2, context=1000),
    "deepseek_v2_bias": shrink(CONFIGS["deepseek_v2"], batch=1, context=200, with_bias=True),
    "qwen25_7b_q4": shrink(CONFIGS["qwen25_7b"], batch=2, context=300, q_len=4),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_decode_step_parity(name):
    wl = make_workload(SMALL[name], spare_pages=3)
    prob = GpuProblem(wl)
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(SMALL[name].batch):
        check_sequence(prob, b, name)


@pytest.mark.parametrize("lens", [[1], [64], [65], [4, 128, 129, 63]])
@pytest.mark.parametrize("q_len", [1, 4])
def test_edge_lengths(lens, q_len):
    """Contexts of exactly the new tokens, one full page, one token past a page."""
    lens = [max(L, q_len) for L in lens]
    cfg = shrink(CONFIGS["qwen3_30b_a3b"], batch=len(lens), context=max(lens), q_len=q_len,
                 name="edge")
    wl = make_workload(cfg, seq_lens=np.array(lens, dtype=np.int32))
    prob = GpuProblem(wl)
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(len(lens)):
        check_sequence(prob, b, f"lens={lens}")


def test_peaked_softmax_stress():
    """q scaled by 8: a peaked softmax that exercises the running-max updates."""
    cfg = shrink(CONFIGS["deepseek_v2"], batch=2, context=700)
    wl = make_workload(cfg, q_scale=8.0)
    prob = GpuProblem(wl)
    prob.step()
    torch.cuda.synchronize()
    for b in range(2):
        check_sequence(prob, b, "peaked")


@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "hybrid_q4", "deepseek_v2"])
def test_split_invariance(name):
    wl = make_workload(SMALL[name])
    prob = GpuProblem(wl, num_splits=1)
    prob.step()
    o1 = prob.o_latent.float().clone()
    l1 = prob.lse.clone()
    for ns in (2, 7, 0):
        ws = mla.mla_decode_workspace_size(prob.dims, wl.cfg.batch, wl.cfg.q_len, prob.max_seq_len, ns)
        prob.workspace = torch.zeros(ws, dtype=torch.uint8, device="cuda")
        prob.decode_only(num_splits=ns)
        torch.cuda.synchronize()
        err = (prob.o_latent.float() - o1).abs().max().item() / o1.abs().max().item()
        assert err <= 2 ** -7, f"splits={ns}: o_latent differs by {err:.3e}"
        assert (prob.lse - l1).abs().max().item() <= 1e-5


def test_paging_invariance_and_determinism():
    """A different physical page layout gives bitwise identical results."""
    cfg = SMALL["qwen3_30b_a3b"]
    wl = make_workload(cfg, spare_pages=11)
    a = GpuProblem(wl, num_splits=3)
    a.step()
    rng = np.random.default_rng(3)
    perm = rng.permutation(wl.num_pages)
    table2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    b = GpuProblem(wl, num_splits=3, block_table=table2)
    b.step()
    torch.cuda.synchronize()
    assert torch.equal(a.o_latent, b.o_latent)
    assert torch.equal(a.lse, b.lse)
    assert torch.equal(a.o, b.o)
    o_prev = a.o.clone()
    a.step()
    assert torch.equal(a.o, o_prev), "repeated step is not bitwise identical"


def test_bad_page_id_is_flagged_not_faulted():
    cfg = SMALL["qwen25_7b"]
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
    # the other sequences are unaffected
    check_sequence(prob, 0, "bad page, seq 0")
    check_sequence(prob, 2, "bad page, seq 2")


def test_length_beyond_plan_is_flagged():
    cfg = SMALL["qwen25_7b"]
    wl = make_workload(cfg)
    prob = GpuProblem(wl, num_splits=1)
    prob.step()
    lens = wl.seq_lens.copy()
    lens[0] = prob.max_seq_len + 1
    prob.seq_lens = torch.from_numpy(lens).cuda()
    prob.decode_only()
    assert mla.mla_get_device_status(prob.workspace.view(torch.int32)[:1], reset=True) == \
        mla.MLA_ERR_DEVICE_BOUNDS
    check_sequence(prob, 1, "bad length, seq 1")


@pytest.mark.parametrize("name", ["deepseek_v2", "qwen3_30b_a3b", "qwen25_7b_q4", "deepseek_v2_bias"])
def test_one_call_step_equals_four_calls(name):
    """mla_decode_step (the append folded into the absorption) writes the same cache rows and
    the same q_ext, o_latent, lse and o, bit for bit, as the four separate calls."""
    wl = make_workload(SMALL[name], spare_pages=3)
    a = GpuProblem(wl)
    b = GpuProblem(wl)
    a.step()                                   # one call
    mla.mla_cache_append(b.dims, b.c_new, b.k_new, b.cos_q, b.sin_q, b.block_table, b.start_pos,
                         b.cache, dev_error=b.workspace.view(torch.int32)[:1])
    mla.mla_absorb_q(b.dims, b.q_nope, b.q_pe, b.cos_q, b.sin_q, b.w_uk, b.q_ext)
    mla.mla_decode_attn(b.dims, b.q_ext, b.cache, b.block_table, b.seq_lens, b.max_seq_len,
                        b.workspace, b.o_latent, b.lse, causal=wl.cfg.causal)
    mla.mla_out_up(b.dims, b.o_latent, b.w_uv, b.o, bias=b.bias)
    torch.cuda.synchronize()
    assert a.device_status() == mla.MLA_OK and b.device_status() == mla.MLA_OK
    for t in ("q_ext", "o_latent", "lse", "o"):
        assert torch.equal(getattr(a, t), getattr(b, t)), t
    # cache rows: compare as bits (unused rows hold NaN in both)
    assert torch.equal(a.cache.view(torch.int16), b.cache.view(torch.int16))


@pytest.mark.parametrize("name,lens", [
    ("deepseek_v2", [1700, 64, 64, 65, 130, 64, 64, 64]),      # one unit cut into many pieces
    ("qwen3_30b_a3b", [900, 70, 64, 700, 64, 66, 64, 64]),
])
def test_skewed_cut_units(name, lens):
    """Two ranges per unit on average with skewed lengths: units cut into 2..many pieces
    (merged by the merge kernel), against the oracle and against a one-range-per-unit plan
    (no cuts); a second call on the same workspace gives the same bits."""
    cfg = shrink(CONFIGS[name], batch=len(lens), context=max(lens), name="skewed")
    wl = make_workload(cfg, seq_lens=np.array(lens, dtype=np.int32))
    prob = GpuProblem(wl, num_splits=2)
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    for b in range(len(lens)):
        check_sequence(prob, b, f"{name} skewed")
    o2 = prob.o_latent.float().clone()
    l2 = prob.lse.clone()
    prob.decode_only(num_splits=2)          # same workspace again
    torch.cuda.synchronize()
    assert torch.equal(prob.o_latent.float(), o2) and torch.equal(prob.lse, l2)
    ws1 = mla.mla_decode_workspace_size(prob.dims, cfg.batch, cfg.q_len, prob.max_seq_len, 1)
    prob.workspace = torch.zeros(ws1, dtype=torch.uint8, device="cuda")
    prob.decode_only(num_splits=1)
    torch.cuda.synchronize()
    err = (prob.o_latent.float() - o2).abs().max().item() / o2.abs().max().item()
    assert err <= 2 ** -7, err
    assert (prob.lse - l2).abs().max().item() <= 1e-5
