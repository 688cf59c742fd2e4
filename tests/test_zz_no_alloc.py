"""mla_decode_attn_noalloc: decode attention for callers that cannot allocate device memory
when they decode (for example code inside an allocator or memory-pool hook, or a runtime
that fixes its device-memory budget at start-up). It must give the same o_latent and lse
as mla_decode_attn with a caller-provided workspace, call after call, and refuse problems
whose partial results do not fit in its fixed scratch array.

This file is named to be collected last: a run that stops at the first failure has then
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import LSE_TOL, O_TOL, GpuProblem, dims_of, max_rel_err

pytestmark = pytest.mark.gpu

CASES = {
    # ragged lengths: sequences are cut between CTAs, so the merge runs on the scratch
    "qwen3_ragged": shrink(CONFIGS["qwen3_30b_a3b"], batch=6, lens_range=(100, 3000)),
    # four query rows per sequence, causal inside the block
    "hybrid_q4": shrink(CONFIGS["hybrid_1m_q4"], batch=2, context=5000),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_decode(name):
    cfg = CASES[name]
    prob = GpuProblem(make_workload(cfg))
    prob.step()                                    # workspace path: append, absorb, decode
    torch.cuda.synchronize()
    ref_o = prob.o_latent.float().cpu().numpy()
    ref_l = prob.lse.cpu().numpy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):                          # two calls in a row share the scratch
        o = torch.full_like(prob.o_latent, float("nan"))
        lse = torch.full_like(prob.lse, float("nan"))
        mla.mla_decode_attn_noalloc(prob.dims, prob.q_ext, prob.cache, prob.block_table,
                                    prob.seq_lens, prob.max_seq_len, err, o, lse,
                                    causal=cfg.causal)
        torch.cuda.synchronize()
        got_o = o.float().cpu().numpy()
        got_l = lse.cpu().numpy()
        assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_l)), f"call {call}"
        assert max_rel_err(got_o, ref_o) <= O_TOL, f"call {call}: o_latent differs"
        assert float(np.max(np.abs(got_l - ref_l))) <= LSE_TOL, f"call {call}: lse differs"
    assert mla.mla_get_device_status(err) == mla.MLA_OK
    # and the no-allocation output against the fp64 oracle itself, sequence by sequence
    for b in range(cfg.batch):
        ref = prob.oracle(b)
        assert max_rel_err(o[b].float().cpu().numpy(), ref["o_latent"]) <= O_TOL, f"seq {b}"
        assert float(np.max(np.abs(lse[b].cpu().numpy() - ref["lse"]))) <= LSE_TOL, f"seq {b}"


def test_noalloc_refusals_launch_nothing():
    """Host-side refusals of the no-allocation decode: an unsupported page size and a
    missing error word are rejected before anything is launched (the pointers here are not
    device memory, so only calls that return before a launch may use them). The automatic
    plan of the benchmark shapes fits the scratch: with bf16 partial outputs it holds at
    most 148 one-CTA ranges of up to 64 rows, or 74 two-CTA ranges of 128 rows, each
    x 2 slots x r <= 512 bf16 = 19.4 MB of partials, plus 4 bytes per sequence."""
    cfg = CONFIGS["deepseek_v2"]
    dims = dims_of(cfg)
    fake = ctypes.c_void_p(0x10000)
    st = mla.lib().mla_decode_attn_noalloc(ctypes.byref(dims_of(cfg.with_(page_size=32))), fake,
                                           fake, 100000, fake, 128, fake, 4, 1, 512, 1, fake,
                                           fake, fake, None)
    assert st == mla.MLA_ERR_UNSUPPORTED
    st = mla.lib().mla_decode_attn_noalloc(ctypes.byref(dims), fake, fake, 100000, fake, 128,
                                           fake, 4, 1, 512, 1, None, fake, fake, None)
    assert st == mla.MLA_ERR_INVALID_ARG            # the error word is required
    scratch = 32 << 20                              # MLA_NOALLOC_SCRATCH_BYTES
    for batch in (64, 256, 4096):
        assert 0 < mla.mla_decode_workspace_size(dims, batch, 1, cfg.context, 0) <= scratch
