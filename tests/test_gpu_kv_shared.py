"""The single-latent K = V form (nanowhale-100m page) on the GPU against the fp64 oracle
``kv_shared_reference``: query rotation, decode over whole cache rows (key = value), and
the inverse rotation of the output, at the parity tolerances (2e-2 * max|ref| on o, 1e-3 on
lse); plus the full benchmark size on sampled sequences."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import LSE_TOL, O_TOL, GpuProblem, max_rel_err

pytestmark = pytest.mark.gpu

NW = CONFIGS["nanowhale_kv_shared"]
CASES = {
    "nanowhale_small": shrink(NW, batch=3, context=777),
    "nanowhale_ragged_q4": shrink(NW, batch=3, lens_range=(4, 600), q_len=4),
    "nanowhale_q4_noncausal": shrink(NW, batch=2, context=300, q_len=4, causal=False),
}


def _check(prob: GpuProblem, b: int, what: str):
    import oracle.mla_oracle as O  # test infrastructure only
    wl, cfg = prob.wl, prob.cfg
    c_kv, k_r = wl.context(b)
    ref = O.kv_shared_reference(wl.q_nope[b], wl.q_pe[b], c_kv, k_r[:, 0, :], wl.theta[0],
                                wl.query_positions()[b], cfg.softmax_scale, causal=cfg.causal)
    o = prob.o_kv[b].float().cpu().numpy()
    lse = prob.lse_kv[b].cpu().numpy()
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), f"{what} seq {b}: non-finite"
    e_o = max_rel_err(o, ref["o"])
    e_l = float(np.max(np.abs(lse - ref["lse"])))
    assert e_o <= O_TOL, f"{what} seq {b}: o rel err {e_o:.3e}"
    assert e_l <= LSE_TOL, f"{what} seq {b}: lse err {e_l:.3e}"
    # the rotary dims alone are checked too (they carry the inverse rotation)
    dn = cfg.kv_lora_rank
    e_r = float(np.max(np.abs(o[..., dn:] - ref["o"][..., dn:]))) / float(np.max(np.abs(ref["o"])))
    assert e_r <= O_TOL, f"{what} seq {b}: rotary dims err {e_r:.3e}"


@pytest.mark.parametrize("splits", [1, 0])
@pytest.mark.parametrize("name", sorted(CASES))
def test_kv_shared_parity(name, splits):
    cfg = CASES[name]
    prob = GpuProblem(make_workload(cfg, spare_pages=2), num_splits=splits)
    prob.kv_shared_step()
    torch.cuda.synchronize()
    assert mla.mla_get_device_status(prob.ws_kv.view(torch.int32)[:1]) == mla.MLA_OK
    for b in range(cfg.batch):
        _check(prob, b, name)


def test_kv_shared_full_size_sampled():
    prob = GpuProblem(make_workload(NW))
    prob.kv_shared_step()
    torch.cuda.synchronize()
    assert mla.mla_get_device_status(prob.ws_kv.view(torch.int32)[:1]) == mla.MLA_OK
    assert bool(torch.isfinite(prob.o_kv.float()).all())
    for b in (0, NW.batch // 2, NW.batch - 1):
        _check(prob, b, "nanowhale full size")


def test_kv_shared_rotation_round_trip():
    """Query rotation then output rotation at the same positions returns the input within
    two bf16 roundings (the rotation is orthogonal)."""
    cfg = CASES["nanowhale_small"]
    prob = GpuProblem(make_workload(cfg))
    x = torch.randn(cfg.batch, 1, cfg.num_heads, cfg.row_width, device="cuda").to(torch.bfloat16)
    y, z = torch.empty_like(x), torch.empty_like(x)
    mla.mla_kv_shared_query(prob.dims, x, prob.cos_q, prob.sin_q, y)
    mla.mla_kv_shared_output(prob.dims, y, prob.cos_q, prob.sin_q, z)
    torch.cuda.synchronize()
    r = cfg.kv_lora_rank
    assert torch.equal(z[..., :r], x[..., :r])
    assert float((z.float() - x.float()).abs().max()) <= 2 ** -6 * float(x.float().abs().max())
