"""mla_absorb_q and mla_out_up on the GPU against the oracle's fp64 definitions
(the q_absorb einsum and einsum (5) of the DeepSeek-V2 page)."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
import oracle.mla_oracle as O
from mla_inputs import CONFIGS, make_workload, shrink
from tests.gpu_harness import dims_of, max_rel_err

pytestmark = pytest.mark.gpu

# fp32 accumulation, bf16 output: one rounding of the result plus bf16 inputs
PROJ_TOL = 1e-2

CASES = {
    "tiny": CONFIGS["tiny"],
    "qwen25_7b": shrink(CONFIGS["qwen25_7b"], batch=5, context=100),
    "deepseek_v2": shrink(CONFIGS["deepseek_v2"], batch=64, context=100),
    "qwen3_30b_a3b": shrink(CONFIGS["qwen3_30b_a3b"], batch=128, context=100),
    "hybrid_q4": shrink(CONFIGS["hybrid_1m_q4"], batch=3, context=100),
    "deepseek_v2_rows200": shrink(CONFIGS["deepseek_v2"], batch=200, context=100),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_absorb_q(name):
    cfg = CASES[name]
    wl = make_workload(cfg)
    dims = dims_of(cfg)
    B, q, H, D, r = cfg.batch, cfg.q_len, cfg.num_heads, cfg.row_width, cfg.kv_lora_rank
    qpos = wl.query_positions()
    cos, sin = wl.rope_table(qpos)
    q_ext = torch.full((B, q, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    mla.mla_absorb_q(dims, wl.q_nope.cuda(), wl.q_pe.cuda(), torch.from_numpy(cos).cuda(),
                     torch.from_numpy(sin).cuda(), wl.w_uk.cuda(), q_ext)
    got = q_ext.float().cpu().numpy()
    G, dr = cfg.num_kv_groups, cfg.rope_dim
    g_of = O.group_of_head(H, G)
    for b in range(B):
        q_c, q_rot = O.absorb_reference(wl.q_nope[b], wl.q_pe[b], wl.w_uk, wl.theta, qpos[b], G)
        assert max_rel_err(got[b, :, :, :r], q_c) <= PROJ_TOL
        for h in range(H):
            for g in range(G):
                sl = got[b, :, h, r + g * dr: r + (g + 1) * dr]
                if g == g_of[h]:
                    assert np.max(np.abs(sl - q_rot[:, h])) <= 2 ** -7 * np.max(np.abs(q_rot)) + 1e-6
                else:
                    assert np.all(sl == 0.0)


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("with_bias", [False, True])
def test_out_up(name, with_bias):
    cfg = CASES[name].with_(with_bias=with_bias)
    wl = make_workload(cfg)
    dims = dims_of(cfg)
    B, q, H, r, dv = cfg.batch, cfg.q_len, cfg.num_heads, cfg.kv_lora_rank, cfg.v_head_dim
    g = torch.Generator().manual_seed(7)
    o_lat = (torch.randn(B, q, H, r, generator=g) / np.sqrt(r)).to(torch.bfloat16)
    o = torch.full((B, q, H, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    mla.mla_out_up(dims, o_lat.cuda(), wl.w_uv.cuda(), o,
                   bias=None if wl.bias is None else wl.bias.cuda())
    ref = O.out_up_reference(o_lat, wl.w_uv, wl.bias)
    assert max_rel_err(o.float().cpu().numpy(), ref) <= PROJ_TOL


def test_packed_kv_b_proj_view():
    """W_UK and W_UV taken straight from a kv_b_proj weight viewed as [H, d_n + d_v, r]."""
    cfg = CASES["deepseek_v2"]
    wl = make_workload(cfg)
    dims = dims_of(cfg)
    H, dn, dv, r = cfg.num_heads, cfg.qk_nope_dim, cfg.v_head_dim, cfg.kv_lora_rank
    kvb = torch.cat([wl.w_uk, wl.w_uv], dim=1).contiguous().cuda()          # [H, d_n + d_v, r]
    B, q, D = cfg.batch, cfg.q_len, cfg.row_width
    cos, sin = wl.rope_table(wl.query_positions())
    q_ext = torch.empty((B, q, H, D), dtype=torch.bfloat16, device="cuda")
    mla.mla_absorb_q(dims, wl.q_nope.cuda(), wl.q_pe.cuda(), torch.from_numpy(cos).cuda(),
                     torch.from_numpy(sin).cuda(), kvb, q_ext, w_uk_head_stride=(dn + dv) * r)
    q_ext2 = torch.empty_like(q_ext)
    mla.mla_absorb_q(dims, wl.q_nope.cuda(), wl.q_pe.cuda(), torch.from_numpy(cos).cuda(),
                     torch.from_numpy(sin).cuda(), wl.w_uk.cuda(), q_ext2)
    assert torch.equal(q_ext, q_ext2)
    o_lat = q_ext[..., :r].contiguous()
    o1 = torch.empty((B, q, H, dv), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    # W_UV of head h starts d_n * r elements into head h's packed block
    mla.mla_out_up(dims, o_lat, kvb.view(-1)[dn * r:], o1, w_uv_head_stride=(dn + dv) * r)
    mla.mla_out_up(dims, o_lat, wl.w_uv.cuda(), o2)
    assert torch.equal(o1, o2)


def _offset_copy(t: torch.Tensor) -> torch.Tensor:
    """The same values in a contiguous tensor whose start is one element past an aligned
    allocation (so 2 or 4 bytes off every wider boundary)."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    out = buf[1:].view(t.shape)
    out.copy_(t)
    return out


@pytest.mark.parametrize("name", ["deepseek_v2", "qwen3_30b_a3b", "hybrid_q4"])
def test_absorb_rope_unaligned_inputs(name):
    """q_pe, cos and sin off their vector alignment take the scalar rotary path; q_ext is
    bit-identical to the aligned call's."""
    cfg = CASES[name]
    wl = make_workload(cfg)
    dims = dims_of(cfg)
    B, q, H, D = cfg.batch, cfg.q_len, cfg.num_heads, cfg.row_width
    cos, sin = wl.rope_table(wl.query_positions())
    q_pe, cos_t, sin_t = wl.q_pe.cuda(), torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda()
    outs = []
    for qp, c, s in ((q_pe, cos_t, sin_t),
                     (_offset_copy(q_pe), _offset_copy(cos_t), _offset_copy(sin_t))):
        q_ext = torch.full((B, q, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        mla.mla_absorb_q(dims, wl.q_nope.cuda(), qp, c, s, wl.w_uk.cuda(), q_ext)
        outs.append(q_ext.view(torch.int16).cpu())
    assert torch.equal(outs[0], outs[1])
