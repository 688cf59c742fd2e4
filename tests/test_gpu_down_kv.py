"""mla_down_kv_append: the KV down-projection of new tokens written straight into the paged
cache by one tcgen05 GEMM.

* The projection (its optional kv_out) against the fp64 oracle ``down_kv_reference``: each
  element within one bf16 rounding (2^-8 relative) plus 1e-3 of accumulation slack.
* The cache bytes against the unfused path: mla_cache_append of the same projected values
  (this call's kv_out) must give bit-identical caches (the append itself is pinned
  bit-exact against the oracle's byte-level emulation in test_gpu_append.py).
* The sum over the model width is split across the CTAs of a cluster and added in a fixed
  order: two calls give the same bits.
* Then the decode over that cache against the decode oracle fed the oracle's own projection.
"""
import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_down_kv_inputs, make_workload, shrink
from tests.gpu_harness import dims_of

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": CONFIGS["tiny"],
    "qwen25_7b": shrink(CONFIGS["qwen25_7b"], batch=5, context=300),
    "deepseek_v2": shrink(CONFIGS["deepseek_v2"], batch=3, context=200),
    "qwen3_30b_a3b": shrink(CONFIGS["qwen3_30b_a3b"], batch=70, lens_range=(5, 400)),
    "hybrid": shrink(CONFIGS["hybrid_1m_q4"], batch=3, context=130),
    "nanowhale": shrink(CONFIGS["nanowhale_kv_shared"], batch=4, context=100),
}


def _run(cfg, n_new, spare=2):
    wl = make_workload(cfg, spare_pages=spare)
    dims = dims_of(cfg)
    B, D = cfg.batch, cfg.row_width
    hidden, w_dkv = make_down_kv_inputs(cfg, n_new)
    start = (wl.seq_lens - n_new).astype(np.int32)
    pos = start[:, None] + np.arange(n_new)[None, :]
    cos, sin = wl.rope_table(pos)
    dev = "cuda"
    t = dict(hidden=hidden.to(dev), w=w_dkv.to(dev), cos=torch.from_numpy(cos).to(dev),
             sin=torch.from_numpy(sin).to(dev), table=torch.from_numpy(wl.block_table).to(dev),
             start=torch.from_numpy(start).to(dev))
    cache = torch.full((wl.num_pages, cfg.page_size, D), float("nan"), dtype=torch.bfloat16,
                       device=dev)
    kv_out = torch.full((B, n_new, D), float("nan"), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.mla_down_kv_append(dims, t["hidden"], t["w"], t["cos"], t["sin"], t["table"], t["start"],
                           cache, dev_error=err, kv_out=kv_out)
    torch.cuda.synchronize()
    return wl, dims, hidden, w_dkv, t, cache, kv_out, err


def _new_rows(wl, cfg, cache, n_new):
    """The cache rows of the n_new appended tokens of every sequence, [B, n_new, D] (float)."""
    out = []
    for b in range(cfg.batch):
        L = int(wl.seq_lens[b])
        pos = np.arange(L - n_new, L)
        pages = torch.from_numpy(wl.block_table[b, pos // cfg.page_size].astype(np.int64)).cuda()
        rows = torch.from_numpy(pos % cfg.page_size).cuda()
        out.append(cache[pages, rows].float().cpu().numpy())
    return np.stack(out)


def _check_projection(cfg, hidden, w_dkv, kv_out):
    import oracle.mla_oracle as O  # test infrastructure only
    c_ref, k_ref = O.down_kv_reference(hidden, w_dkv, cfg.kv_lora_rank, cfg.num_kv_groups,
                                       cfg.rope_dim)
    ref = np.concatenate([c_ref, k_ref.reshape(k_ref.shape[:-2] + (-1,))], axis=-1)
    got = kv_out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    bound = 2.0 ** -8 * np.abs(ref) + 1e-3
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{int(bad.sum())} elements off, worst {np.max(np.abs(got - ref)):.3e}"
    return ref


@pytest.mark.parametrize("n_new", [1, 4])
@pytest.mark.parametrize("name", sorted(CASES))
def test_down_kv_append(name, n_new):
    cfg = CASES[name]
    wl, dims, hidden, w_dkv, t, cache, kv_out, err = _run(cfg, n_new)
    assert mla.mla_get_device_status(err) == mla.MLA_OK
    _check_projection(cfg, hidden, w_dkv, kv_out)
    # the unfused path on the same projected values gives the same cache bytes
    r = cfg.kv_lora_rank
    ref_cache = torch.full_like(cache, float("nan"))
    k_r = kv_out[..., r:].reshape(cfg.batch, n_new, cfg.num_kv_groups, cfg.rope_dim).contiguous()
    # (the unfused append of this call's own projection)
    mla.mla_cache_append(dims, kv_out[..., :r].contiguous(), k_r, t["cos"], t["sin"], t["table"],
                         t["start"], ref_cache, dev_error=err)
    torch.cuda.synchronize()
    assert torch.equal(cache.view(torch.int16), ref_cache.view(torch.int16))


def test_down_kv_without_kv_out_and_bad_page():
    """kv_out is optional; a page id out of range is flagged and that token skipped."""
    import oracle.mla_oracle as O  # test infrastructure only
    cfg = CASES["deepseek_v2"]
    n = 4
    wl, dims, hidden, w_dkv, t, cache, kv_out, err = _run(cfg, n)
    c_ref, _ = O.down_kv_reference(hidden, w_dkv, cfg.kv_lora_rank, cfg.num_kv_groups,
                                   cfg.rope_dim)
    r = cfg.kv_lora_rank
    cache2 = torch.full_like(cache, float("nan"))
    mla.mla_down_kv_append(dims, t["hidden"], t["w"], t["cos"], t["sin"], t["table"], t["start"],
                           cache2, dev_error=err)
    torch.cuda.synchronize()
    got = _new_rows(wl, cfg, cache2, n)[..., :r]
    assert np.all(np.abs(got - c_ref) <= 2.0 ** -8 * np.abs(c_ref) + 1e-3)
    bad = wl.block_table.copy()
    last = (int(wl.seq_lens[1]) - 1) // cfg.page_size
    bad[1, last] = wl.num_pages + 7
    cache3 = torch.full_like(cache, float("nan"))
    mla.mla_down_kv_append(dims, t["hidden"], t["w"], t["cos"], t["sin"],
                           torch.from_numpy(bad).cuda(), t["start"], cache3, dev_error=err)
    assert mla.mla_get_device_status(err, reset=True) == mla.MLA_ERR_DEVICE_BOUNDS
    # sequences 0 and 2 are written
    got3 = _new_rows(wl, cfg, cache3, n)
    for b in (0, 2):
        assert np.all(np.abs(got3[b, :, :r] - c_ref[b]) <= 2.0 ** -8 * np.abs(c_ref[b]) + 1e-3)


@pytest.mark.parametrize("name", ["deepseek_v2", "qwen3_30b_a3b"])
def test_down_kv_deterministic(name):
    """Two calls on the same inputs give the same projection and cache bits (the split sum
    is added in a fixed order)."""
    cfg = CASES[name]
    _, dims, _, _, t, cache, kv_out, err = _run(cfg, 4)
    cache2 = torch.full_like(cache, float("nan"))
    kv2 = torch.full_like(kv_out, float("nan"))
    mla.mla_down_kv_append(dims, t["hidden"], t["w"], t["cos"], t["sin"], t["table"], t["start"],
                           cache2, dev_error=err, kv_out=kv2)
    torch.cuda.synchronize()
    assert mla.mla_get_device_status(err) == mla.MLA_OK
    assert torch.equal(kv_out.view(torch.int16), kv2.view(torch.int16))
    assert torch.equal(cache.view(torch.int16), cache2.view(torch.int16))


def test_down_kv_full_size_deepseek():
    """The DeepSeek-V2 shape at its bench size: 64 new tokens of width 5120 into a 576-wide row."""
    cfg = CONFIGS["deepseek_v2"].with_(context=128)
    wl, dims, hidden, w_dkv, t, cache, kv_out, err = _run(cfg, 1)
    assert mla.mla_get_device_status(err) == mla.MLA_OK
    _check_projection(cfg, hidden, w_dkv, kv_out)


def test_decode_after_fused_append():
    """The decode over a cache whose last tokens came from the fused projection matches the
    decode oracle given the oracle's own fp64 projection of those tokens (rounded to bf16)."""
    import oracle.mla_oracle as O  # test infrastructure only
    from tests.gpu_harness import GpuProblem, LSE_TOL, O_TOL, max_rel_err
    cfg = shrink(CONFIGS["qwen3_30b_a3b"], batch=3, lens_range=(70, 500), q_len=4)
    wl = make_workload(cfg)
    prob = GpuProblem(wl)                 # cache holds every token but the last q
    hidden, w_dkv = make_down_kv_inputs(cfg, cfg.q_len)
    c_new, k_new = O.down_kv_reference(hidden, w_dkv, cfg.kv_lora_rank, cfg.num_kv_groups,
                                       cfg.rope_dim)
    mla.mla_down_kv_append(prob.dims, hidden.cuda(), w_dkv.cuda(), prob.cos_q, prob.sin_q,
                           prob.block_table, prob.start_pos, prob.cache, dev_error=prob.err)
    mla.mla_absorb_q(prob.dims, prob.q_nope, prob.q_pe, prob.cos_q, prob.sin_q, prob.w_uk,
                     prob.q_ext)
    prob.decode_only()
    mla.mla_out_up(prob.dims, prob.o_latent, prob.w_uv, prob.o, bias=prob.bias)
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    q = cfg.q_len
    for b in range(cfg.batch):
        c_kv, k_r = wl.context(b)
        c_kv = c_kv.clone()
        k_r = k_r.clone()
        c_kv[-q:] = torch.from_numpy(c_new[b]).to(torch.bfloat16)
        k_r[-q:] = torch.from_numpy(k_new[b]).to(torch.bfloat16)
        ref = O.mla_decode_reference(wl.q_nope[b], wl.q_pe[b], c_kv, k_r, wl.w_uk, wl.w_uv,
                                     wl.bias, wl.theta, wl.query_positions()[b],
                                     cfg.softmax_scale, causal=cfg.causal)
        assert max_rel_err(prob.o[b].float().cpu().numpy(), ref["o"]) <= O_TOL
        assert float(np.max(np.abs(prob.lse[b].cpu().numpy() - ref["lse"]))) <= LSE_TOL
