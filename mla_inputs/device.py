"""One MLA decode problem resident on the GPU, built from a seeded workload.

The cache is pre-filled through the library's mla_cache_append (every context token but
the last q); ``step()`` then runs the decode step through the library's four calls
(append of the last q tokens, absorb, decode, out_up), all on the C ABI. Unwritten cache
slots hold bf16 NaN so that a kernel reading past a context shows up as NaN.

Used by the GPU tests (which add the oracle comparisons) and by bench.py. It holds no
arithmetic of the method: every step runs in the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

import head_latent_attention_attn_b200 as mla

from .configs import MLAConfig
from .generate import Workload


def dims_of(cfg: MLAConfig) -> mla.MlaDims:
    return mla.make_dims(cfg.num_heads, cfg.num_kv_groups, cfg.kv_lora_rank, cfg.qk_nope_dim,
                         cfg.rope_dim, cfg.v_head_dim, cfg.page_size, cfg.softmax_scale)


class DeviceProblem:
    def __init__(self, wl: Workload, num_splits: int = 0, device: str = "cuda",
                 fill_nan: bool = True, block_table: np.ndarray = None):
        cfg = wl.cfg
        self.wl, self.cfg = wl, cfg
        self.dev = torch.device(device)
        self.dims = dims_of(cfg)
        self.num_splits = num_splits
        B, q, H, G = cfg.batch, cfg.q_len, cfg.num_heads, cfg.num_kv_groups
        r, dr, D, ps = cfg.kv_lora_rank, cfg.rope_dim, cfg.row_width, cfg.page_size
        dev = self.dev
        fill = float("nan") if fill_nan else 0.0
        self.cache = torch.full((wl.num_pages, ps, D), fill, dtype=torch.bfloat16, device=dev)
        table = wl.block_table if block_table is None else block_table
        self.block_table = torch.from_numpy(np.ascontiguousarray(table)).to(dev)
        self.seq_lens = torch.from_numpy(wl.seq_lens).to(dev)
        self.max_seq_len = int(wl.seq_lens.max())
        self.w_uk = wl.w_uk.to(dev)
        self.w_uv = wl.w_uv.to(dev)
        self.bias = None if wl.bias is None else wl.bias.to(dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

        c_new = torch.empty((B, q, r), dtype=torch.bfloat16)
        k_new = torch.empty((B, q, G, dr), dtype=torch.bfloat16)
        lens = [int(L) for L in wl.seq_lens]
        # uniform lengths: one batched append (few launches); ragged: one per sequence
        batched = len(set(lens)) == 1 and lens[0] > q and B * lens[0] * D * 2 <= (2 << 30)
        if batched:
            n = lens[0] - q
            ctx = [wl.context(b) for b in range(B)]
            cos, sin = wl.rope_table(np.arange(n))
            cos = np.broadcast_to(cos[None], (B,) + cos.shape)
            sin = np.broadcast_to(sin[None], (B,) + sin.shape)
            mla.mla_cache_append(self.dims, torch.stack([c[:n] for c, _ in ctx]).to(dev),
                                 torch.stack([k[:n] for _, k in ctx]).to(dev),
                                 torch.from_numpy(np.array(cos, order="C")).to(dev),
                                 torch.from_numpy(np.array(sin, order="C")).to(dev),
                                 self.block_table, torch.zeros(B, dtype=torch.int32, device=dev),
                                 self.cache, dev_error=self.err)
            for b, (c_kv, k_r) in enumerate(ctx):
                c_new[b] = c_kv[n:n + q]
                k_new[b] = k_r[n:n + q]
            del ctx
        for b in range(0 if not batched else B, B):
            c_kv, k_r = wl.context(b)
            L = lens[b]
            n = L - q
            if n > 0:
                cos, sin = wl.rope_table(np.arange(n))
                mla.mla_cache_append(self.dims, c_kv[None, :n].to(dev).contiguous(),
                                     k_r[None, :n].to(dev).contiguous(),
                                     torch.from_numpy(cos[None]).to(dev),
                                     torch.from_numpy(sin[None]).to(dev),
                                     self.block_table[b:b + 1],
                                     torch.zeros(1, dtype=torch.int32, device=dev), self.cache,
                                     dev_error=self.err)
            c_new[b] = c_kv[L - q:L]
            k_new[b] = k_r[L - q:L]
        qpos = wl.query_positions()
        cos_q, sin_q = wl.rope_table(qpos)
        self.c_new = c_new.to(dev)
        self.k_new = k_new.to(dev)
        self.cos_q = torch.from_numpy(cos_q).to(dev)
        self.sin_q = torch.from_numpy(sin_q).to(dev)
        self.start_pos = torch.from_numpy((wl.seq_lens - q).astype(np.int32)).to(dev)
        self.q_nope = wl.q_nope.to(dev)
        self.q_pe = wl.q_pe.to(dev)
        self.q_ext = torch.empty((B, q, H, D), dtype=torch.bfloat16, device=dev)
        self.o_latent = torch.empty((B, q, H, r), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, q, H), dtype=torch.float32, device=dev)
        self.o = torch.empty((B, q, H, cfg.v_head_dim), dtype=torch.bfloat16, device=dev)
        ws = mla.mla_decode_workspace_size(self.dims, B, q, self.max_seq_len, num_splits)
        assert ws > 0
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def step(self, stream=None) -> None:
        mla.mla_decode_step(self.dims, c_kv_new=self.c_new, k_r_new=self.k_new,
                            cos_new=self.cos_q, sin_new=self.sin_q, start_pos=self.start_pos,
                            q_nope=self.q_nope, q_pe=self.q_pe, cos_q=self.cos_q,
                            sin_q=self.sin_q, w_uk=self.w_uk, w_uv=self.w_uv, bias=self.bias,
                            cache=self.cache, block_table=self.block_table,
                            seq_lens=self.seq_lens, max_seq_len=self.max_seq_len,
                            q_ext=self.q_ext, workspace=self.workspace, o_latent=self.o_latent,
                            lse=self.lse, o=self.o, causal=self.cfg.causal,
                            num_splits=self.num_splits, stream=stream)

    def step_four_calls(self, stream=None) -> None:
        """The same decode step as four library calls: append, absorb, decode (+ merge),
        up-projection."""
        mla.mla_cache_append(self.dims, self.c_new, self.k_new, self.cos_q, self.sin_q,
                             self.block_table, self.start_pos, self.cache,
                             dev_error=self.workspace.view(torch.int32)[:1], stream=stream)
        mla.mla_absorb_q(self.dims, self.q_nope, self.q_pe, self.cos_q, self.sin_q, self.w_uk,
                         self.q_ext, stream=stream)
        mla.mla_decode_attn(self.dims, self.q_ext, self.cache, self.block_table, self.seq_lens,
                            self.max_seq_len, self.workspace, self.o_latent, self.lse,
                            causal=self.cfg.causal, num_splits=self.num_splits, stream=stream)
        mla.mla_out_up(self.dims, self.o_latent, self.w_uv, self.o, bias=self.bias, stream=stream)

    def decode_only(self, num_splits=None) -> None:
        ns = self.num_splits if num_splits is None else num_splits
        mla.mla_decode_attn(self.dims, self.q_ext, self.cache, self.block_table, self.seq_lens,
                            self.max_seq_len, self.workspace, self.o_latent, self.lse,
                            causal=self.cfg.causal, num_splits=ns)

    def device_status(self) -> int:
        a = mla.mla_get_device_status(self.err)
        b = mla.mla_get_device_status(self.workspace.view(torch.int32)[:1])
        return max(a, b)

    # ---- the single-latent K = V form ------------------------------------------------------
    def kv_shared_step(self, stream=None, num_splits=None) -> None:
        """One step of the K = V form on this problem's cache: append the last q tokens,
        rotate the query's rotary slice, decode over whole rows (the decode view of the dims)
        and rotate the output's rotary slice back. Output in ``self.o_kv`` [B, q, H, D]."""
        cfg = self.cfg
        B, q, H, D = cfg.batch, cfg.q_len, cfg.num_heads, cfg.row_width
        ns = self.num_splits if num_splits is None else num_splits
        if not hasattr(self, "o_kv"):
            self.kv_dims = mla.mla_kv_shared_decode_dims(self.dims)
            self.q_kv = torch.cat([self.q_nope, self.q_pe], dim=-1).contiguous()
            self.q_ext_kv = torch.empty((B, q, H, D), dtype=torch.bfloat16, device=self.dev)
            self.o_lat_kv = torch.empty((B, q, H, D), dtype=torch.bfloat16, device=self.dev)
            self.lse_kv = torch.empty((B, q, H), dtype=torch.float32, device=self.dev)
            self.o_kv = torch.empty((B, q, H, D), dtype=torch.bfloat16, device=self.dev)
            ws = mla.mla_decode_workspace_size(self.kv_dims, B, q, self.max_seq_len, ns)
            self.ws_kv = torch.zeros(ws, dtype=torch.uint8, device=self.dev)
        mla.mla_cache_append(self.dims, self.c_new, self.k_new, self.cos_q, self.sin_q,
                             self.block_table, self.start_pos, self.cache,
                             dev_error=self.ws_kv.view(torch.int32)[:1], stream=stream)
        mla.mla_kv_shared_query(self.dims, self.q_kv, self.cos_q, self.sin_q, self.q_ext_kv,
                                stream=stream)
        mla.mla_decode_attn(self.kv_dims, self.q_ext_kv, self.cache, self.block_table,
                            self.seq_lens, self.max_seq_len, self.ws_kv, self.o_lat_kv,
                            self.lse_kv, causal=cfg.causal, num_splits=ns, stream=stream)
        mla.mla_kv_shared_output(self.dims, self.o_lat_kv, self.cos_q, self.sin_q, self.o_kv,
                                 stream=stream)
