"""Python binding of libmla.so, the B200 (sm_100a) weight-absorbed MLA decode library.

The functions here carry the C ABI's names (include/mla.h) and only marshal arguments:
they check torch tensors' device, dtype, contiguity and shapes, take their data
pointers and the current CUDA stream, and call the library. Every step of the decode
path runs in the library's CUDA kernels; there is no other implementation. If the
library is not built, every call raises ``MlaError``.

Decode step, in the absorbed order of the DeepSeek-V2 MLA page ("Matrix absorption"):
    mla_cache_append -> mla_absorb_q -> mla_decode_attn -> mla_out_up
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_BOUNDS = 5
MLA_ERR_DEVICE_TIMEOUT = 6
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
                3: "MLA_ERR_WORKSPACE", 4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_BOUNDS",
                6: "MLA_ERR_DEVICE_TIMEOUT"}

# Public C symbols (kept in sync with include/mla.h; a CPU test checks both ways).
C_SYMBOLS = ("mla_row_width", "mla_status_string", "mla_cache_append", "mla_absorb_q",
             "mla_decode_workspace_size", "mla_decode_attn", "mla_out_up",
             "mla_get_device_status", "mla_decode_attn_noalloc", "mla_selftest_wait_timeout",
             "mla_kv_shared_decode_dims", "mla_kv_shared_query", "mla_kv_shared_output",
             "mla_down_kv_append", "mla_out_proj_workspace_size",
             "mla_out_proj", "mla_decode_step")


class MlaError(RuntimeError):
    def __init__(self, msg: str, status: int = MLA_ERR_CUDA):
        super().__init__(msg)
        self.status = status


class MlaDims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("num_kv_groups", ctypes.c_int32),
                ("kv_lora_rank", ctypes.c_int32), ("qk_nope_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("v_head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]

    @property
    def row_width(self) -> int:
        return self.kv_lora_rank + self.num_kv_groups * self.rope_dim


def make_dims(num_heads: int, num_kv_groups: int, kv_lora_rank: int, qk_nope_dim: int,
              rope_dim: int, v_head_dim: int, page_size: int, softmax_scale: float) -> MlaDims:
    return MlaDims(num_heads, num_kv_groups, kv_lora_rank, qk_nope_dim, rope_dim, v_head_dim,
                   page_size, softmax_scale)


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """Load libmla.so (raises MlaError when it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise MlaError(f"{LIB_PATH} is missing: build it with "
                       "`python -m head_latent_attention_attn_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    D = ctypes.POINTER(MlaDims)
    L.mla_row_width.argtypes = [D]
    L.mla_row_width.restype = _I32
    L.mla_status_string.argtypes = [_I32]
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_cache_append.argtypes = [D, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _P, _I64, _P, _P]
    L.mla_cache_append.restype = _I32
    L.mla_absorb_q.argtypes = [D, _P, _P, _P, _P, _P, _I64, _I32, _I32, _P, _P]
    L.mla_absorb_q.restype = _I32
    L.mla_decode_workspace_size.argtypes = [D, _I32, _I32, _I32, _I32]
    L.mla_decode_workspace_size.restype = ctypes.c_size_t
    L.mla_decode_attn.argtypes = [D, _P, _P, _I64, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                  _P, ctypes.c_size_t, _P, _P, _P]
    L.mla_decode_attn.restype = _I32
    L.mla_out_up.argtypes = [D, _P, _P, _I64, _P, _I32, _P, _P]
    L.mla_out_up.restype = _I32
    L.mla_get_device_status.argtypes = [_P, _I32, _P]
    L.mla_get_device_status.restype = _I32
    L.mla_decode_attn_noalloc.argtypes = [D, _P, _P, _I64, _P, _I32, _P, _I32, _I32, _I32, _I32,
                                          _P, _P, _P, _P]
    L.mla_decode_attn_noalloc.restype = _I32
    L.mla_selftest_wait_timeout.argtypes = [_P, _P]
    L.mla_selftest_wait_timeout.restype = _I32
    L.mla_kv_shared_decode_dims.argtypes = [D, D]
    L.mla_kv_shared_decode_dims.restype = _I32
    for fn in (L.mla_kv_shared_query, L.mla_kv_shared_output):
        fn.argtypes = [D, _P, _P, _P, _I32, _I32, _P, _P]
        fn.restype = _I32
    L.mla_down_kv_append.argtypes = [D, _P, _I32, _P, _P, _P, _P, _I32, _P, _I32, _I32, _P,
                                     _I64, _P, _P, _P]
    L.mla_down_kv_append.restype = _I32
    L.mla_out_proj_workspace_size.argtypes = [D, _I32, _I32]
    L.mla_out_proj_workspace_size.restype = ctypes.c_size_t
    L.mla_out_proj.argtypes = [D, _P, _P, _I64, _P, _P, _P, _I32, _I32, _P, ctypes.c_size_t, _P,
                               _P, _P]
    L.mla_out_proj.restype = _I32
    L.mla_decode_step.argtypes = [D, _P, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P, _I64, _P, _I64,
                                  _P, _P, _I64, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _P,
                                  _P, ctypes.c_size_t, _P, _P, _P, _P]
    L.mla_decode_step.restype = _I32
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, what: str) -> None:
    if status != MLA_OK:
        raise MlaError(f"{what}: {STATUS_NAMES.get(status, status)}", status)


def _need(t, name: str, dtype, shape=None, cuda: bool = True) -> None:
    if not isinstance(t, torch.Tensor):
        raise MlaError(f"{name} must be a torch.Tensor", MLA_ERR_INVALID_ARG)
    if cuda and t.device.type != "cuda":
        raise MlaError(f"{name} must be on a CUDA device", MLA_ERR_INVALID_ARG)
    if t.dtype != dtype:
        raise MlaError(f"{name} must be {dtype}, got {t.dtype}", MLA_ERR_INVALID_ARG)
    if not t.is_contiguous():
        raise MlaError(f"{name} must be contiguous", MLA_ERR_INVALID_ARG)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise MlaError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}",
                       MLA_ERR_INVALID_ARG)


def mla_row_width(dims: MlaDims) -> int:
    return int(lib().mla_row_width(ctypes.byref(dims)))


def mla_cache_append(dims: MlaDims, c_kv, k_r, rope_cos, rope_sin, block_table, start_pos,
                     cache, dev_error=None, stream=None) -> None:
    """Write c_kv [B, n, r] and RoPE(k_r [B, n, G, d_r]) into cache [P, ps, D] in place."""
    B, n = c_kv.shape[0], c_kv.shape[1]
    G, dr, r = dims.num_kv_groups, dims.rope_dim, dims.kv_lora_rank
    _need(c_kv, "c_kv", torch.bfloat16, (B, n, r))
    if dr > 0:
        _need(k_r, "k_r", torch.bfloat16, (B, n, G, dr))
        _need(rope_cos, "rope_cos", torch.float32, (B, n, G, dr // 2))
        _need(rope_sin, "rope_sin", torch.float32, (B, n, G, dr // 2))
    _need(block_table, "block_table", torch.int32)
    _need(start_pos, "start_pos", torch.int32, (B,))
    _need(cache, "cache", torch.bfloat16)
    if cache.dim() != 3 or cache.shape[1] != dims.page_size or cache.shape[2] != dims.row_width:
        raise MlaError(f"cache shape {tuple(cache.shape)} does not match dims", MLA_ERR_INVALID_ARG)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise MlaError("block_table must be [B, max_pages]", MLA_ERR_INVALID_ARG)
    if dev_error is not None:
        _need(dev_error, "dev_error", torch.int32)
    st = lib().mla_cache_append(ctypes.byref(dims), _ptr(c_kv), _ptr(k_r if dr > 0 else None),
                                _ptr(rope_cos if dr > 0 else None),
                                _ptr(rope_sin if dr > 0 else None), _ptr(block_table),
                                block_table.shape[1], _ptr(start_pos), B, n, _ptr(cache),
                                cache.shape[0], _ptr(dev_error), _stream(stream))
    _check(st, "mla_cache_append")


def mla_down_kv_append(dims: MlaDims, hidden, w_dkv, rope_cos, rope_sin, block_table,
                       start_pos, cache, dev_error=None, kv_out=None, stream=None) -> None:
    """[c_kv ; k_r] = w_dkv @ hidden (bf16) for hidden [B, n, hidden_dim], written into cache
    [P, ps, D] exactly as mla_cache_append would; kv_out [B, n, D] optionally receives the
    projection before the rotation."""
    B, n, hid = hidden.shape
    G, dr, D = dims.num_kv_groups, dims.rope_dim, dims.row_width
    _need(hidden, "hidden", torch.bfloat16)
    _need(w_dkv, "w_dkv", torch.bfloat16, (D, hid))
    if dr > 0:
        _need(rope_cos, "rope_cos", torch.float32, (B, n, G, dr // 2))
        _need(rope_sin, "rope_sin", torch.float32, (B, n, G, dr // 2))
    _need(block_table, "block_table", torch.int32)
    _need(start_pos, "start_pos", torch.int32, (B,))
    _need(cache, "cache", torch.bfloat16)
    if cache.dim() != 3 or cache.shape[1] != dims.page_size or cache.shape[2] != D:
        raise MlaError(f"cache shape {tuple(cache.shape)} does not match dims", MLA_ERR_INVALID_ARG)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise MlaError("block_table must be [B, max_pages]", MLA_ERR_INVALID_ARG)
    if dev_error is not None:
        _need(dev_error, "dev_error", torch.int32)
    if kv_out is not None:
        _need(kv_out, "kv_out", torch.bfloat16, (B, n, D))
    st = lib().mla_down_kv_append(ctypes.byref(dims), _ptr(hidden), hid, _ptr(w_dkv),
                                  _ptr(rope_cos if dr > 0 else None),
                                  _ptr(rope_sin if dr > 0 else None), _ptr(block_table),
                                  block_table.shape[1], _ptr(start_pos), B, n, _ptr(cache),
                                  cache.shape[0], _ptr(dev_error), _ptr(kv_out),
                                  _stream(stream))
    _check(st, "mla_down_kv_append")


def mla_absorb_q(dims: MlaDims, q_nope, q_pe, rope_cos, rope_sin, w_uk, q_ext,
                 w_uk_head_stride: Optional[int] = None, stream=None) -> None:
    """q_ext [B, q, H, D] = [W_UK^T q_nope ; RoPE(q_pe) in its group's slot, zeros elsewhere]."""
    B, q = q_nope.shape[0], q_nope.shape[1]
    H, G, dr = dims.num_heads, dims.num_kv_groups, dims.rope_dim
    _need(q_nope, "q_nope", torch.bfloat16, (B, q, H, dims.qk_nope_dim))
    if dr > 0:
        _need(q_pe, "q_pe", torch.bfloat16, (B, q, H, dr))
        _need(rope_cos, "rope_cos", torch.float32, (B, q, G, dr // 2))
        _need(rope_sin, "rope_sin", torch.float32, (B, q, G, dr // 2))
    _need(q_ext, "q_ext", torch.bfloat16, (B, q, H, dims.row_width))
    if w_uk_head_stride is None:
        _need(w_uk, "w_uk", torch.bfloat16, (H, dims.qk_nope_dim, dims.kv_lora_rank))
        w_uk_head_stride = dims.qk_nope_dim * dims.kv_lora_rank
    else:
        _need(w_uk, "w_uk", torch.bfloat16)
    st = lib().mla_absorb_q(ctypes.byref(dims), _ptr(q_nope), _ptr(q_pe if dr > 0 else None),
                            _ptr(rope_cos if dr > 0 else None), _ptr(rope_sin if dr > 0 else None),
                            _ptr(w_uk), int(w_uk_head_stride), B, q, _ptr(q_ext),
                            _stream(stream))
    _check(st, "mla_absorb_q")


def mla_decode_workspace_size(dims: MlaDims, batch: int, q_len: int, max_seq_len: int,
                              num_splits: int = 0) -> int:
    return int(lib().mla_decode_workspace_size(ctypes.byref(dims), batch, q_len, max_seq_len,
                                               num_splits))


def mla_decode_attn(dims: MlaDims, q_ext, cache, block_table, seq_lens, max_seq_len: int,
                    workspace, o_latent, lse, causal: bool = True, num_splits: int = 0,
                    stream=None) -> None:
    """o_latent [B, q, H, r] (bf16) and lse [B, q, H] (fp32) of the absorbed attention."""
    B, q = q_ext.shape[0], q_ext.shape[1]
    H, r = dims.num_heads, dims.kv_lora_rank
    _need(q_ext, "q_ext", torch.bfloat16, (B, q, H, dims.row_width))
    _need(cache, "cache", torch.bfloat16)
    if cache.dim() != 3 or cache.shape[1] != dims.page_size or cache.shape[2] != dims.row_width:
        raise MlaError(f"cache shape {tuple(cache.shape)} does not match dims", MLA_ERR_INVALID_ARG)
    _need(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise MlaError("block_table must be [B, max_pages]", MLA_ERR_INVALID_ARG)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(o_latent, "o_latent", torch.bfloat16, (B, q, H, r))
    _need(lse, "lse", torch.float32, (B, q, H))
    _need(workspace, "workspace", torch.uint8)
    st = lib().mla_decode_attn(ctypes.byref(dims), _ptr(q_ext), _ptr(cache), cache.shape[0],
                               _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, q,
                               int(max_seq_len), 1 if causal else 0, int(num_splits),
                               _ptr(workspace), workspace.numel(), _ptr(o_latent), _ptr(lse),
                               _stream(stream))
    _check(st, "mla_decode_attn")


def mla_decode_attn_noalloc(dims: MlaDims, q_ext, cache, block_table, seq_lens,
                            max_seq_len: int, dev_error, o_latent, lse, causal: bool = True,
                            stream=None) -> None:
    """mla_decode_attn without a workspace, for callers that cannot allocate device memory
    at decode time: the library's own fixed scratch array stands in for the workspace.
    Calls that overlap on the GPU share that array and must not be issued."""
    B, q = q_ext.shape[0], q_ext.shape[1]
    H, r = dims.num_heads, dims.kv_lora_rank
    _need(q_ext, "q_ext", torch.bfloat16, (B, q, H, dims.row_width))
    _need(cache, "cache", torch.bfloat16)
    if cache.dim() != 3 or cache.shape[1] != dims.page_size or cache.shape[2] != dims.row_width:
        raise MlaError(f"cache shape {tuple(cache.shape)} does not match dims", MLA_ERR_INVALID_ARG)
    _need(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise MlaError("block_table must be [B, max_pages]", MLA_ERR_INVALID_ARG)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(dev_error, "dev_error", torch.int32)
    _need(o_latent, "o_latent", torch.bfloat16, (B, q, H, r))
    _need(lse, "lse", torch.float32, (B, q, H))
    st = lib().mla_decode_attn_noalloc(ctypes.byref(dims), _ptr(q_ext), _ptr(cache), cache.shape[0],
                                       _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B,
                                       q, int(max_seq_len), 1 if causal else 0, _ptr(dev_error),
                                       _ptr(o_latent), _ptr(lse), _stream(stream))
    _check(st, "mla_decode_attn_noalloc")


def mla_out_up(dims: MlaDims, o_latent, w_uv, o, bias=None,
               w_uv_head_stride: Optional[int] = None, stream=None) -> None:
    """o [rows, H, d_v] = W_UV o_latent (+ bias); o_latent is [rows, H, r] (any leading shape)."""
    H, r, dv = dims.num_heads, dims.kv_lora_rank, dims.v_head_dim
    _need(o_latent, "o_latent", torch.bfloat16)
    if o_latent.shape[-2:] != (H, r):
        raise MlaError("o_latent must end in [H, r]", MLA_ERR_INVALID_ARG)
    rows = o_latent.numel() // (H * r)
    _need(o, "o", torch.bfloat16)
    if o.numel() != rows * H * dv:
        raise MlaError("o must hold rows * H * d_v elements", MLA_ERR_INVALID_ARG)
    if w_uv_head_stride is None:
        _need(w_uv, "w_uv", torch.bfloat16, (H, dv, r))
        w_uv_head_stride = dv * r
    else:
        _need(w_uv, "w_uv", torch.bfloat16)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (H, dv))
    st = lib().mla_out_up(ctypes.byref(dims), _ptr(o_latent), _ptr(w_uv), int(w_uv_head_stride),
                          _ptr(bias), rows, _ptr(o), _stream(stream))
    _check(st, "mla_out_up")


def mla_kv_shared_decode_dims(dims: MlaDims) -> MlaDims:
    """Decode view of a K = V layout: the whole cache row is the latent (rank D, no rotary
    slot), so mla_decode_attn with these dims returns o_latent = sum_l p_l row_l."""
    out = MlaDims()
    _check(lib().mla_kv_shared_decode_dims(ctypes.byref(dims), ctypes.byref(out)),
           "mla_kv_shared_decode_dims")
    return out


def _kv_shared_rotate(fn, what, dims: MlaDims, x, rope_cos, rope_sin, out, stream) -> None:
    B, q = x.shape[0], x.shape[1]
    D = dims.row_width
    _need(x, what + " input", torch.bfloat16, (B, q, dims.num_heads, D))
    _need(out, what + " output", torch.bfloat16, (B, q, dims.num_heads, D))
    _need(rope_cos, "rope_cos", torch.float32, (B, q, 1, dims.rope_dim // 2))
    _need(rope_sin, "rope_sin", torch.float32, (B, q, 1, dims.rope_dim // 2))
    _check(fn(ctypes.byref(dims), _ptr(x), _ptr(rope_cos), _ptr(rope_sin), B, q, _ptr(out),
              _stream(stream)), what)


def mla_kv_shared_query(dims: MlaDims, q, rope_cos, rope_sin, q_ext, stream=None) -> None:
    """q_ext [B, q, H, D] = q with its last d_r dims rotated to the query positions."""
    _kv_shared_rotate(lib().mla_kv_shared_query, "mla_kv_shared_query", dims, q, rope_cos,
                      rope_sin, q_ext, stream)


def mla_kv_shared_output(dims: MlaDims, o_latent, rope_cos, rope_sin, o, stream=None) -> None:
    """o [B, q, H, D] = o_latent with its last d_r dims rotated back from the query positions."""
    _kv_shared_rotate(lib().mla_kv_shared_output, "mla_kv_shared_output", dims, o_latent,
                      rope_cos, rope_sin, o, stream)


def mla_out_proj_workspace_size(dims: MlaDims, hidden: int, rows: int) -> int:
    return int(lib().mla_out_proj_workspace_size(ctypes.byref(dims), int(hidden), int(rows)))


def mla_out_proj(dims: MlaDims, o_latent, w_uv, w_o, workspace, o, u, bias_v=None, bias_o=None,
                 w_uv_head_stride: Optional[int] = None, stream=None) -> None:
    """o [rows, H, d_v] = W_UV o_latent (+ bias_v) and u [rows, hidden] = W_o o (+ bias_o) in
    one kernel; w_o is [hidden, H * d_v]; workspace a zeroed uint8 CUDA tensor."""
    H, r, dv = dims.num_heads, dims.kv_lora_rank, dims.v_head_dim
    _need(o_latent, "o_latent", torch.bfloat16)
    if o_latent.shape[-2:] != (H, r):
        raise MlaError("o_latent must end in [H, r]", MLA_ERR_INVALID_ARG)
    rows = o_latent.numel() // (H * r)
    _need(w_o, "w_o", torch.bfloat16)
    if w_o.dim() != 2 or w_o.shape[1] != H * dv:
        raise MlaError("w_o must be [hidden, H * d_v]", MLA_ERR_INVALID_ARG)
    hidden = w_o.shape[0]
    _need(o, "o", torch.bfloat16)
    if o.numel() != rows * H * dv:
        raise MlaError("o must hold rows * H * d_v elements", MLA_ERR_INVALID_ARG)
    _need(u, "u", torch.bfloat16)
    if u.numel() != rows * hidden:
        raise MlaError("u must hold rows * hidden elements", MLA_ERR_INVALID_ARG)
    if w_uv_head_stride is None:
        _need(w_uv, "w_uv", torch.bfloat16, (H, dv, r))
        w_uv_head_stride = dv * r
    else:
        _need(w_uv, "w_uv", torch.bfloat16)
    if bias_v is not None:
        _need(bias_v, "bias_v", torch.bfloat16, (H, dv))
    if bias_o is not None:
        _need(bias_o, "bias_o", torch.bfloat16, (hidden,))
    _need(workspace, "workspace", torch.uint8)
    st = lib().mla_out_proj(ctypes.byref(dims), _ptr(o_latent), _ptr(w_uv), int(w_uv_head_stride),
                            _ptr(bias_v), _ptr(w_o), _ptr(bias_o), hidden, rows, _ptr(workspace),
                            workspace.numel(), _ptr(o), _ptr(u), _stream(stream))
    _check(st, "mla_out_proj")


def mla_get_device_status(dev_error, reset: bool = False, stream=None) -> int:
    """Synchronise and read a device error word (an int32 tensor, or a decode workspace)."""
    if dev_error.device.type != "cuda":
        raise MlaError("dev_error must be on a CUDA device", MLA_ERR_INVALID_ARG)
    return int(lib().mla_get_device_status(_ptr(dev_error), 1 if reset else 0, _stream(stream)))


def mla_selftest_wait_timeout(dev_error, stream=None) -> None:
    """Launch the device error path's self-test: a bounded wait that nothing completes, which
    sets MLA_DEVERR_TIMEOUT in dev_error (an int32 CUDA tensor) after about 2 s."""
    _need(dev_error, "dev_error", torch.int32)
    _check(lib().mla_selftest_wait_timeout(_ptr(dev_error), _stream(stream)),
           "mla_selftest_wait_timeout")


def mla_decode_step(dims: MlaDims, *, c_kv_new, k_r_new, cos_new, sin_new, start_pos,
                    q_nope, q_pe, cos_q, sin_q, w_uk, w_uv, bias, cache, block_table, seq_lens,
                    max_seq_len: int, q_ext, workspace, o_latent, lse, o, causal: bool = True,
                    num_splits: int = 0, w_uk_head_stride: Optional[int] = None,
                    w_uv_head_stride: Optional[int] = None, stream=None) -> None:
    """One decode step in one library call (append, absorb, attention, up-projection): the
    outputs of mla_cache_append, mla_absorb_q, mla_decode_attn and mla_out_up on the same
    arguments. c_kv_new [B, n, r] / k_r_new [B, n, G, d_r] are the appended tokens."""
    B, q = q_nope.shape[0], q_nope.shape[1]
    n = c_kv_new.shape[1]
    H, G, dr, r, dv, D = (dims.num_heads, dims.num_kv_groups, dims.rope_dim, dims.kv_lora_rank,
                          dims.v_head_dim, dims.row_width)
    _need(c_kv_new, "c_kv_new", torch.bfloat16, (B, n, r))
    _need(q_nope, "q_nope", torch.bfloat16, (B, q, H, dims.qk_nope_dim))
    if dr > 0:
        _need(k_r_new, "k_r_new", torch.bfloat16, (B, n, G, dr))
        _need(cos_new, "cos_new", torch.float32, (B, n, G, dr // 2))
        _need(sin_new, "sin_new", torch.float32, (B, n, G, dr // 2))
        _need(q_pe, "q_pe", torch.bfloat16, (B, q, H, dr))
        _need(cos_q, "cos_q", torch.float32, (B, q, G, dr // 2))
        _need(sin_q, "sin_q", torch.float32, (B, q, G, dr // 2))
    _need(start_pos, "start_pos", torch.int32, (B,))
    if w_uk_head_stride is None:
        _need(w_uk, "w_uk", torch.bfloat16, (H, dims.qk_nope_dim, r))
        w_uk_head_stride = dims.qk_nope_dim * r
    else:
        _need(w_uk, "w_uk", torch.bfloat16)
    if w_uv_head_stride is None:
        _need(w_uv, "w_uv", torch.bfloat16, (H, dv, r))
        w_uv_head_stride = dv * r
    else:
        _need(w_uv, "w_uv", torch.bfloat16)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (H, dv))
    _need(cache, "cache", torch.bfloat16)
    if cache.dim() != 3 or cache.shape[1] != dims.page_size or cache.shape[2] != D:
        raise MlaError(f"cache shape {tuple(cache.shape)} does not match dims", MLA_ERR_INVALID_ARG)
    _need(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise MlaError("block_table must be [B, max_pages]", MLA_ERR_INVALID_ARG)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(q_ext, "q_ext", torch.bfloat16, (B, q, H, D))
    _need(workspace, "workspace", torch.uint8)
    _need(o_latent, "o_latent", torch.bfloat16, (B, q, H, r))
    _need(lse, "lse", torch.float32, (B, q, H))
    _need(o, "o", torch.bfloat16, (B, q, H, dv))
    st = lib().mla_decode_step(
        ctypes.byref(dims), _ptr(c_kv_new), _ptr(k_r_new if dr > 0 else None),
        _ptr(cos_new if dr > 0 else None), _ptr(sin_new if dr > 0 else None), _ptr(start_pos), n,
        _ptr(q_nope), _ptr(q_pe if dr > 0 else None), _ptr(cos_q if dr > 0 else None),
        _ptr(sin_q if dr > 0 else None), _ptr(w_uk), int(w_uk_head_stride), _ptr(w_uv),
        int(w_uv_head_stride), _ptr(bias), _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, q, int(max_seq_len), 1 if causal else 0,
        int(num_splits), _ptr(q_ext), _ptr(workspace), workspace.numel(), _ptr(o_latent),
        _ptr(lse), _ptr(o), _stream(stream))
    _check(st, "mla_decode_step")


__all__ = ["MlaDims", "MlaError", "make_dims", "lib", "mla_row_width", "mla_cache_append",
           "mla_absorb_q", "mla_decode_workspace_size", "mla_decode_attn", "mla_out_up",
           "mla_decode_attn_noalloc", "mla_kv_shared_decode_dims", "mla_kv_shared_query",
           "mla_kv_shared_output", "mla_down_kv_append",
           "mla_out_proj_workspace_size",
           "mla_out_proj", "mla_get_device_status", "mla_decode_step", "C_SYMBOLS", "STATUS_NAMES"]
