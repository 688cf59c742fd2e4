"""mla_out_proj: einsum (5) and einsum (6) of the DeepSeek-V2 page in one cooperative kernel,
against the fp64 oracle (out_up_reference then o_proj_reference) at the parity tolerance
(2e-2 * max|ref|), with and without biases, over one and several row tiles, at the
DeepSeek-V2 benchmark size; calls in a row on one workspace (its counters must be left
clear) and bitwise determinism (fixed-order reduction of the K splits)."""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_o_proj_inputs, make_workload, shrink
from tests.gpu_harness import O_TOL, dims_of, max_rel_err

pytestmark = pytest.mark.gpu


def _inputs(cfg, rows, bias):
    wl = make_workload(cfg.with_(context=64, lens_range=None, batch=1))
    g = torch.Generator("cpu")
    g.manual_seed(cfg.seed + 5)
    o_lat = (torch.randn(rows, cfg.num_heads, cfg.kv_lora_rank, generator=g) /
             np.sqrt(cfg.kv_lora_rank)).to(torch.bfloat16)
    bias_v = wl.bias if bias else None
    if bias and bias_v is None:
        bias_v = (torch.randn(cfg.num_heads, cfg.v_head_dim, generator=g) * 0.1).to(torch.bfloat16)
    w_o, bias_o = make_o_proj_inputs(cfg, with_bias=bias)
    return o_lat, wl.w_uv, bias_v, w_o, bias_o


def _ref(cfg, o_lat, w_uv, bias_v, w_o, bias_o):
    import oracle.mla_oracle as O  # test infrastructure only
    o = O.out_up_reference(o_lat, w_uv, bias_v)
    w_heads = O.as_f64(w_o).T.reshape(cfg.num_heads, cfg.v_head_dim, -1)    # [H, d_v, hidden]
    return o, O.o_proj_reference(o, w_heads, bias_o)


def _counters_bytes(cfg, rows):
    """Bytes of the workspace's counters (error word, CTA count, per-head and per-tile
    counters), which every call must leave zero; the fp32 partials follow them."""
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nr = 16 if rows <= 16 else 32 if rows <= 32 else 64 if rows <= 64 else 128
    n_nt = (rows + nr - 1) // nr
    n_mt = (cfg.hidden_size + 127) // 128
    tile_off = a256(256 + cfg.num_heads * 4)
    return a256(tile_off + n_mt * n_nt * 4)


def _run(cfg, rows, bias, calls=2):
    """`calls` calls on one workspace; call k uses o_latent * (-1)^k, so a counter left set
    by one call (stage B not waiting for stage A) would show up in the next one's output."""
    o_lat, w_uv, bias_v, w_o, bias_o = _inputs(cfg, rows, bias)
    dims = dims_of(cfg)
    dev = "cuda"
    ws = torch.zeros(mla.mla_out_proj_workspace_size(dims, cfg.hidden_size, rows),
                     dtype=torch.uint8, device=dev)
    t = [x.to(dev) if x is not None else None for x in (o_lat, w_uv, bias_v, w_o, bias_o)]
    outs = []
    for k in range(calls):
        sign = -1.0 if k % 2 else 1.0
        o = torch.full((rows, cfg.num_heads, cfg.v_head_dim), float("nan"), dtype=torch.bfloat16,
                       device=dev)
        u = torch.full((rows, cfg.hidden_size), float("nan"), dtype=torch.bfloat16, device=dev)
        mla.mla_out_proj(dims, (t[0] * sign).contiguous(), t[1], t[3], ws, o, u, bias_v=t[2],
                         bias_o=t[4])
        torch.cuda.synchronize()
        assert mla.mla_get_device_status(ws.view(torch.int32)[:1]) == mla.MLA_OK
        assert int(ws[:_counters_bytes(cfg, rows)].count_nonzero()) == 0, "counters left set"
        outs.append((sign, o, u))
    return (o_lat, w_uv, bias_v, w_o, bias_o), outs


CASES = {
    "deepseek_rows64": (CONFIGS["deepseek_v2"], 64, False),
    "deepseek_rows5_bias": (CONFIGS["deepseek_v2"], 5, True),
    "hybrid_rows200_bias": (CONFIGS["hybrid_1m_q4"], 200, True),
    "qwen3_rows128": (CONFIGS["qwen3_30b_a3b"], 128, False),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_out_proj_parity(name):
    cfg, rows, bias = CASES[name]
    ins, outs = _run(cfg, rows, bias, calls=3)
    o_lat, w_uv, bias_v, w_o, bias_o = ins
    for sign, o, u in outs:
        o_ref, u_ref = _ref(cfg, o_lat.float() * sign, w_uv, bias_v, w_o, bias_o)
        got_o = o.float().cpu().numpy()
        got_u = u.float().cpu().numpy()
        assert np.all(np.isfinite(got_o)) and np.all(np.isfinite(got_u))
        assert max_rel_err(got_o, o_ref) <= O_TOL, f"{name}: o {max_rel_err(got_o, o_ref):.3e}"
        assert max_rel_err(got_u, u_ref) <= O_TOL, f"{name}: u {max_rel_err(got_u, u_ref):.3e}"
    # deterministic: the same inputs give the same bits (calls 0 and 2)
    assert torch.equal(outs[0][2], outs[2][2]) and torch.equal(outs[0][1], outs[2][1])


def test_out_proj_matches_out_up():
    """Stage (5) of the fused kernel gives exactly mla_out_up's o (same fp32 sums per feature)."""
    cfg, rows, bias = CONFIGS["deepseek_v2"], 64, True
    ins, outs = _run(cfg, rows, bias, calls=1)
    o_lat, w_uv, bias_v = ins[0].cuda(), ins[1].cuda(), ins[2].cuda()
    o2 = torch.empty_like(outs[0][1])
    mla.mla_out_up(dims_of(cfg), o_lat, w_uv, o2, bias=bias_v)
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], o2)
