"""Seeded synthetic inputs for MLA decode, shared by the oracle tests and the GPU path.

Recipe (all drawn in fp32 from ``torch.Generator('cpu')`` and rounded to bf16):

* every tensor is N(0, 1) / sqrt(its last dimension): c_kv / sqrt(r), k_r / sqrt(d_r),
  q_nope / sqrt(d_n), q_pe / sqrt(d_r), W_UK and W_UV / sqrt(r), bias / sqrt(d_v);
* the main generator is seeded with ``1000 + workload index`` and draws, in this
  order: ragged context lengths, per-group RoPE frequency indices, the physical page
  permutation, W_UK, W_UV, bias, q_nope, q_pe;
* the cached context of sequence b (c_kv and the unrotated k_r of every token) comes
  from its own generator, so any one sequence can be rebuilt without the others;
* token l of a sequence sits at position l; query row i of sequence b sits at
  position L_b - q + i (the last q tokens are the ones appended in the decode step);
* ``identity_weights`` replaces W_UK and W_UV by identity matrices (drawn values unused);
* RoPE frequencies are theta[g, j] = base ** (-2 * idx[g, j] / ref_dim); cos/sin
  tables handed to the GPU are the fp64 cosine/sine of theta * position rounded
  to fp32.

Nothing here implements the attention method itself.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np
import torch

from .configs import MLAConfig


def _randn(gen: torch.Generator, shape, scale_dim: int) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    return (x / math.sqrt(scale_dim)).to(torch.bfloat16)


def _seq_seed(cfg: MLAConfig, b: int) -> int:
    return (cfg.seed * 1_000_003 + 7919 * (b + 1)) % (2 ** 62)


@dataclass
class Workload:
    cfg: MLAConfig
    seq_lens: np.ndarray          # int32 [B], context length after the step's append
    rope_index: np.ndarray        # int64 [G, d_r/2]
    theta: np.ndarray             # float64 [G, d_r/2]
    w_uk: torch.Tensor            # bf16 [H, d_n, r]
    w_uv: torch.Tensor            # bf16 [H, d_v, r]
    bias: Optional[torch.Tensor]  # bf16 [H, d_v] or None
    q_nope: torch.Tensor          # bf16 [B, q, H, d_n]
    q_pe: torch.Tensor            # bf16 [B, q, H, d_r]   (before rotation)
    block_table: np.ndarray       # int32 [B, max_pages]; -1 past the last used page
    num_pages: int
    spare_pages: Tuple[int, ...] = ()
    _ctx_cache: Dict[int, Tuple[torch.Tensor, torch.Tensor]] = field(default_factory=dict)

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    def context(self, b: int, keep: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
        """(c_kv [L_b, r] bf16, k_r [L_b, G, d_r] bf16) of sequence b, unrotated."""
        if b in self._ctx_cache:
            return self._ctx_cache[b]
        cfg = self.cfg
        L = int(self.seq_lens[b])
        g = torch.Generator("cpu")
        g.manual_seed(_seq_seed(cfg, b))
        c_kv = _randn(g, (L, cfg.kv_lora_rank), cfg.kv_lora_rank)
        if cfg.rope_dim > 0:
            k_r = _randn(g, (L, cfg.num_kv_groups, cfg.rope_dim), cfg.rope_dim)
        else:
            k_r = torch.zeros((L, cfg.num_kv_groups, 0), dtype=torch.bfloat16)
        if keep:
            self._ctx_cache[b] = (c_kv, k_r)
        return c_kv, k_r

    def rope_table(self, positions: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
        """fp32 cos/sin tables [*positions.shape, G, d_r/2] for the given positions."""
        ang = np.asarray(positions, dtype=np.float64)[..., None, None] * self.theta
        return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)

    def query_positions(self) -> np.ndarray:
        """int64 [B, q]: position of each query row."""
        q = self.cfg.q_len
        return self.seq_lens.astype(np.int64)[:, None] - q + np.arange(q)[None, :]


def make_workload(cfg: MLAConfig, q_scale: float = 1.0, spare_pages: int = 0,
                  seq_lens: Optional[np.ndarray] = None) -> Workload:
    """Build the seeded workload for ``cfg``.

    ``q_scale`` multiplies q_nope and q_pe before bf16 rounding (a peaked-softmax
    stress variant); ``spare_pages`` adds physical pages no sequence owns.
    """
    B, q, H, G = cfg.batch, cfg.q_len, cfg.num_heads, cfg.num_kv_groups
    r, dn, dr, dv, ps = cfg.kv_lora_rank, cfg.qk_nope_dim, cfg.rope_dim, cfg.v_head_dim, cfg.page_size
    gen = torch.Generator("cpu")
    gen.manual_seed(cfg.seed)

    if seq_lens is not None:
        lens = np.asarray(seq_lens, dtype=np.int32)
        assert lens.shape == (B,)
    elif cfg.lens_range is not None:
        lo, hi = cfg.lens_range
        lens = torch.randint(lo, hi + 1, (B,), generator=gen).numpy().astype(np.int32)
    else:
        lens = np.full((B,), cfg.context, dtype=np.int32)

    half = dr // 2
    if cfg.rope_index_pool > 0:
        idx = np.stack([np.sort(torch.randperm(cfg.rope_index_pool, generator=gen)[:half].numpy())
                        for _ in range(G)]).astype(np.int64)
    else:
        idx = np.tile(np.arange(half, dtype=np.int64), (G, 1))
    theta = cfg.rope_base ** (-2.0 * idx.astype(np.float64) / float(cfg.rope_ref_dim))

    pages_per_seq = [(int(L) + ps - 1) // ps for L in lens]
    used = int(sum(pages_per_seq))
    num_pages = used + spare_pages
    max_pages = max(pages_per_seq)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    if cfg.contiguous:
        phys = np.arange(num_pages, dtype=np.int64)
    else:
        phys = torch.randperm(num_pages, generator=gen).numpy()
    k = 0
    for b, n in enumerate(pages_per_seq):
        table[b, :n] = phys[k:k + n]
        k += n
    spare = tuple(int(p) for p in phys[used:])

    w_uk = _randn(gen, (H, dn, r), r)
    w_uv = _randn(gen, (H, dv, r), r)
    if cfg.identity_weights:
        # the special case in which the method is multi-query attention over c_kv itself
        assert dn == r and dv == r, "identity weights need d_n = d_v = r"
        w_uk = torch.eye(r, dtype=torch.bfloat16).expand(H, r, r).contiguous()
        w_uv = w_uk.clone()
    bias = _randn(gen, (H, dv), dv) if cfg.with_bias else None
    qn = torch.randn(B, q, H, dn, generator=gen, dtype=torch.float32) / math.sqrt(dn)
    qp = torch.randn(B, q, H, dr, generator=gen, dtype=torch.float32) / math.sqrt(max(dr, 1))
    q_nope = (qn * q_scale).to(torch.bfloat16)
    q_pe = (qp * q_scale).to(torch.bfloat16)
    return Workload(cfg=cfg, seq_lens=lens, rope_index=idx, theta=theta, w_uk=w_uk, w_uv=w_uv,
                    bias=bias, q_nope=q_nope, q_pe=q_pe, block_table=table,
                    num_pages=num_pages, spare_pages=spare)


def make_down_kv_inputs(cfg: MLAConfig, n_new: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Inputs of the KV down-projection for ``cfg``: hidden states [B, n_new, hidden] ~ N(0, 1)
    and the stacked projection [r + G*d_r, hidden] ~ N(0, 1) / sqrt(hidden) (down_kv rows,
    then each group's k_r_proj rows), both rounded to bf16, from their own seeded generator."""
    gen = torch.Generator("cpu")
    gen.manual_seed(cfg.seed * 31 + 17)
    hidden = torch.randn(cfg.batch, n_new, cfg.hidden_size, generator=gen).to(torch.bfloat16)
    w_dkv = _randn(gen, (cfg.row_width, cfg.hidden_size), cfg.hidden_size)
    return hidden, w_dkv


def make_o_proj_inputs(cfg: MLAConfig, with_bias: bool = False):
    """The output projection for ``cfg``: w_o [hidden, H * d_v] ~ N(0, 1) / sqrt(H * d_v) (row k
    holds W_o[h, d, k] at column h * d_v + d) and, if asked, bias [hidden] ~ N(0, 1) / sqrt(hidden),
    bf16, from their own seeded generator."""
    gen = torch.Generator("cpu")
    gen.manual_seed(cfg.seed * 37 + 23)
    K = cfg.num_heads * cfg.v_head_dim
    w_o = _randn(gen, (cfg.hidden_size, K), K)
    bias = _randn(gen, (cfg.hidden_size,), cfg.hidden_size) if with_bias else None
    return w_o, bias
