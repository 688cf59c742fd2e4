"""mla_cache_append on the GPU: bit-exact against the oracle's byte-level emulation."""
import zlib

import numpy as np
import pytest
import torch

import head_latent_attention_attn_b200 as mla
import oracle.mla_oracle as O
from mla_inputs import CONFIGS
from tests.gpu_harness import dims_of

pytestmark = pytest.mark.gpu


def _case(cfg, B, n, npages, seed, maxp=None):
    rng = np.random.default_rng(seed)
    ps, r, G, dr, D = cfg.page_size, cfg.kv_lora_rank, cfg.num_kv_groups, cfg.rope_dim, cfg.row_width
    start = rng.integers(0, 3 * ps, size=B).astype(np.int32)
    need = [(int(s) + n + ps - 1) // ps for s in start]
    maxp = maxp or max(need)
    perm = rng.permutation(npages)
    table = np.full((B, maxp), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        table[b, :need[b]] = perm[k:k + need[b]]
        k += need[b]
    assert k <= npages
    c_bits = rng.integers(0, 2 ** 16, size=(B, n, r), dtype=np.uint64).astype(np.uint16)
    k_f = (rng.standard_normal((B, n, G, dr)) * 3).astype(np.float32)
    k_bits = torch.from_numpy(k_f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ang = rng.uniform(-40.0, 40.0, size=(B, n, G, dr // 2))
    cos32, sin32 = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    cache_bits = np.full((npages, ps, D), 0xABCD, dtype=np.uint16)
    return start, table, c_bits, k_bits, cos32, sin32, cache_bits


def _to_dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("name", ["tiny", "qwen25_7b", "deepseek_v2", "qwen3_30b_a3b", "hybrid_1m_q4"])
@pytest.mark.parametrize("n", [1, 4, 67])
def test_append_bit_exact(name, n):
    cfg = CONFIGS[name]
    B = 5
    start, table, c_bits, k_bits, cos32, sin32, cache_bits = _case(cfg, B, n, 64, seed=zlib.crc32(f"{name}-{n}".encode()) % 1000)
    want = O.cache_append_emulate(cache_bits, c_bits, k_bits, cos32, sin32, table, start, cfg.page_size)
    cache = _to_dev_bf16(cache_bits.copy())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_cache_append(dims_of(cfg), _to_dev_bf16(c_bits), _to_dev_bf16(k_bits),
                         torch.from_numpy(cos32).cuda(), torch.from_numpy(sin32).cuda(),
                         torch.from_numpy(table).cuda(), torch.from_numpy(start).cuda(), cache,
                         dev_error=err)
    got = cache.view(torch.int16).cpu().numpy().view(np.uint16)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} mismatching elements, first {bad[:4].tolist()}"
    assert mla.mla_get_device_status(err) == mla.MLA_OK


def test_append_out_of_range_page_is_flagged_and_skipped():
    cfg = CONFIGS["qwen25_7b"]
    B, n = 3, 4
    start, table, c_bits, k_bits, cos32, sin32, cache_bits = _case(cfg, B, n, 32, seed=5)
    bad_table = table.copy()
    bad_table[1, start[1] // cfg.page_size] = 32 + 7          # outside [0, num_pages)
    ok_rows = [0, 2]
    want = O.cache_append_emulate(cache_bits, c_bits[ok_rows], k_bits[ok_rows], cos32[ok_rows],
                                  sin32[ok_rows], table[ok_rows], start[ok_rows], cfg.page_size)
    # tokens of sequence 1 that do not fall on the corrupted page are still written
    keep = (start[1] + np.arange(n)) // cfg.page_size != start[1] // cfg.page_size
    if keep.any():
        want = O.cache_append_emulate(want, c_bits[1:2, keep], k_bits[1:2, keep], cos32[1:2, keep],
                                      sin32[1:2, keep], table[1:2],
                                      np.array([start[1] + np.nonzero(keep)[0][0]]), cfg.page_size)
    cache = _to_dev_bf16(cache_bits.copy())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_cache_append(dims_of(cfg), _to_dev_bf16(c_bits), _to_dev_bf16(k_bits),
                         torch.from_numpy(cos32).cuda(), torch.from_numpy(sin32).cuda(),
                         torch.from_numpy(bad_table).cuda(), torch.from_numpy(start).cuda(), cache,
                         dev_error=err)
    got = cache.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert mla.mla_get_device_status(err, reset=True) == mla.MLA_ERR_DEVICE_BOUNDS
    assert mla.mla_get_device_status(err) == mla.MLA_OK
