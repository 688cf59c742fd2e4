"""The C ABI without a GPU: every declared symbol is exported, and host-side argument
validation returns the documented status before any CUDA call."""
import ctypes
import os
import re

import pytest

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(mla_\w+)\s*\(", src, flags=re.M))
    return names


def _dims(cfg=None, **kw):
    c = cfg or CONFIGS["deepseek_v2"]
    d = dict(num_heads=c.num_heads, num_kv_groups=c.num_kv_groups, kv_lora_rank=c.kv_lora_rank,
             qk_nope_dim=c.qk_nope_dim, rope_dim=c.rope_dim, v_head_dim=c.v_head_dim,
             page_size=c.page_size, softmax_scale=c.softmax_scale)
    d.update(kw)
    return mla.make_dims(**d)


def test_every_declared_symbol_is_exported(mla_lib):
    declared = _declared_symbols()
    assert declared == set(mla.C_SYMBOLS), declared ^ set(mla.C_SYMBOLS)
    for name in declared:
        assert hasattr(mla_lib, name), name


def test_row_width(mla_lib):
    for c in CONFIGS.values():
        assert mla.mla_row_width(_dims(c)) == c.row_width
    assert mla.mla_row_width(_dims(num_kv_groups=3)) == -1       # 128 % 3 != 0
    assert mla.mla_row_width(_dims(kv_lora_rank=100)) == -1      # not a multiple of 8
    assert mla.mla_row_width(_dims(rope_dim=7)) == -1            # odd rotary dims
    assert mla.mla_row_width(_dims(softmax_scale=0.0)) == -1


def test_status_strings(mla_lib):
    for code, name in mla.STATUS_NAMES.items():
        assert mla_lib.mla_status_string(code).decode() == name


P = ctypes.c_void_p
FAKE = P(0x10000)  # 16-byte-aligned, never dereferenced: validation fails before use


def _append(d, **kw):
    a = dict(c_kv=FAKE, k_r=FAKE, cos=FAKE, sin=FAKE, table=FAKE, maxp=4, start=FAKE, batch=2,
             n=1, cache=FAKE, npages=8, err=None)
    a.update(kw)
    return mla.lib().mla_cache_append(ctypes.byref(d), a["c_kv"], a["k_r"], a["cos"], a["sin"],
                                      a["table"], a["maxp"], a["start"], a["batch"], a["n"],
                                      a["cache"], a["npages"], a["err"], None)


def test_append_validation(mla_lib):
    assert _append(_dims(num_kv_groups=3)) == mla.MLA_ERR_INVALID_ARG
    assert _append(_dims(), c_kv=None) == mla.MLA_ERR_INVALID_ARG
    assert _append(_dims(), k_r=None) == mla.MLA_ERR_INVALID_ARG
    assert _append(_dims(), cache=P(0x10008)) == mla.MLA_ERR_INVALID_ARG   # misaligned
    assert _append(_dims(), batch=-1) == mla.MLA_ERR_INVALID_ARG
    assert _append(_dims(), npages=0) == mla.MLA_ERR_INVALID_ARG
    assert _append(_dims(), batch=0) == mla.MLA_OK                          # nothing to do
    assert _append(_dims(), n=0) == mla.MLA_OK


def _decode(d, **kw):
    a = dict(q=FAKE, cache=FAKE, npages=100, table=FAKE, maxp=4, lens=FAKE, batch=2, qlen=1,
             maxlen=256, causal=1, splits=1, ws=P(0x10000), wsb=1 << 20, o=FAKE, lse=FAKE)
    a.update(kw)
    return mla.lib().mla_decode_attn(ctypes.byref(d), a["q"], a["cache"], a["npages"], a["table"],
                                     a["maxp"], a["lens"], a["batch"], a["qlen"], a["maxlen"],
                                     a["causal"], a["splits"], a["ws"], a["wsb"], a["o"],
                                     a["lse"], None)


def test_decode_validation(mla_lib):
    assert _decode(_dims(page_size=32)) == mla.MLA_ERR_UNSUPPORTED
    assert _decode(_dims(kv_lora_rank=1024)) == mla.MLA_ERR_UNSUPPORTED
    assert _decode(_dims(), qlen=0) == mla.MLA_ERR_INVALID_ARG
    assert _decode(_dims(), maxlen=0) == mla.MLA_ERR_INVALID_ARG
    assert _decode(_dims(), causal=2) == mla.MLA_ERR_INVALID_ARG
    assert _decode(_dims(), lens=None) == mla.MLA_ERR_INVALID_ARG
    assert _decode(_dims(), ws=None) == mla.MLA_ERR_WORKSPACE
    assert _decode(_dims(), ws=P(0x10010)) == mla.MLA_ERR_WORKSPACE          # not 256-aligned
    assert _decode(_dims(), splits=4, wsb=4096) == mla.MLA_ERR_WORKSPACE      # partials need room
    assert _decode(_dims(), batch=0) == mla.MLA_OK


def _step(d, **kw):
    a = dict(c_kv=FAKE, k_r=FAKE, cosn=FAKE, sinn=FAKE, start=FAKE, n=1, qn=FAKE, qpe=FAKE,
             cosq=FAKE, sinq=FAKE, wuk=FAKE, wuks=128 * 512, wuv=FAKE, wuvs=128 * 512, bias=None,
             cache=FAKE, npages=100, table=FAKE, maxp=4, lens=FAKE, batch=2, qlen=1, maxlen=256,
             causal=1, splits=1, qext=FAKE, ws=P(0x10000), wsb=1 << 20, ol=FAKE, lse=FAKE, o=FAKE)
    a.update(kw)
    return mla.lib().mla_decode_step(
        ctypes.byref(d), a["c_kv"], a["k_r"], a["cosn"], a["sinn"], a["start"], a["n"], a["qn"],
        a["qpe"], a["cosq"], a["sinq"], a["wuk"], a["wuks"], a["wuv"], a["wuvs"], a["bias"],
        a["cache"], a["npages"], a["table"], a["maxp"], a["lens"], a["batch"], a["qlen"],
        a["maxlen"], a["causal"], a["splits"], a["qext"], a["ws"], a["wsb"], a["ol"], a["lse"],
        a["o"], None)


def test_decode_step_validation(mla_lib):
    """The one-call step returns the status of the first of its four parts whose arguments
    fail, before anything is launched (FAKE pointers are never dereferenced)."""
    assert _step(_dims(num_kv_groups=3)) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(), c_kv=None) == mla.MLA_ERR_INVALID_ARG               # append
    assert _step(_dims(), npages=0) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(), qn=None) == mla.MLA_ERR_INVALID_ARG                 # absorb
    assert _step(_dims(), wuks=128 * 512 - 8) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(), qext=P(0x10008)) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(page_size=32)) == mla.MLA_ERR_UNSUPPORTED              # decode plan
    assert _step(_dims(), causal=2) == mla.MLA_ERR_INVALID_ARG                # decode
    assert _step(_dims(), lens=None) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(), ws=None) == mla.MLA_ERR_WORKSPACE
    assert _step(_dims(), splits=4, wsb=4096) == mla.MLA_ERR_WORKSPACE
    assert _step(_dims(), wuv=None) == mla.MLA_ERR_INVALID_ARG                # out_up
    assert _step(_dims(), o=P(0x10008)) == mla.MLA_ERR_INVALID_ARG
    assert _step(_dims(), batch=0) == mla.MLA_OK                              # nothing to do


def test_workspace_size(mla_lib):
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # 128 heads, q = 1: one block of 128 query rows per sequence on a cluster of two CTAs
    # that split the latent; 64 units, n ranges (clusters) per unit, two partial slots each
    # (bf16 partial o, fp32 partial lse)
    d = _dims()
    for n in (1, 4):
        ranges = 64 * n
        off = a256(256 + 256 + 64 * 4)                  # error word, range, unit starts
        off = a256(off + ranges * 2 * 128 * 4)          # partial lse
        assert mla.mla_decode_workspace_size(d, 64, 1, 8192, n) == off + ranges * 2 * 128 * 512 * 2
    # 32 heads, q = 1: blocks of 32 rows, one CTA per range
    d32 = _dims(num_heads=32)
    for n in (1, 3):
        ranges = 64 * n
        off = a256(256 + 256 + 64 * 4)
        off = a256(off + ranges * 2 * 32 * 4)
        assert mla.mla_decode_workspace_size(d32, 64, 1, 8192, n) == off + ranges * 2 * 32 * 512 * 2
    # 128 heads of rank 320 (not a multiple of 128): two blocks of 64 rows instead
    d320 = _dims(kv_lora_rank=320)
    off = a256(256 + 256 + 128 * 4)
    off = a256(off + 128 * 2 * 64 * 4)
    assert mla.mla_decode_workspace_size(d320, 64, 1, 8192, 1) == off + 128 * 2 * 64 * 320 * 2
    assert mla.mla_decode_workspace_size(d, 64, 0, 8192, 1) == 0        # invalid q_len
    assert mla.mla_decode_workspace_size(_dims(page_size=16), 1, 1, 64, 1) == 0


def test_absorb_and_out_up_validation(mla_lib):
    L = mla.lib()
    d = _dims()
    st = L.mla_absorb_q(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 4, 1, FAKE, None)
    assert st == mla.MLA_ERR_INVALID_ARG                # head stride < d_n * r
    st = L.mla_absorb_q(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, 128 * 512, 4, 1, FAKE, None)
    assert st == mla.MLA_ERR_INVALID_ARG
    st = L.mla_absorb_q(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 128 * 512, 0, 1, FAKE, None)
    assert st == mla.MLA_OK
    st = L.mla_out_up(ctypes.byref(d), FAKE, FAKE, 128 * 512 + 4, None, 4, FAKE, None)
    assert st == mla.MLA_ERR_INVALID_ARG                # head stride not a multiple of 8
    st = L.mla_out_up(ctypes.byref(d), FAKE, FAKE, 128 * 512, None, 0, FAKE, None)
    assert st == mla.MLA_OK
    assert L.mla_get_device_status(None, 0, None) == mla.MLA_ERR_INVALID_ARG
    assert L.mla_selftest_wait_timeout(None, None) == mla.MLA_ERR_INVALID_ARG   # no launch


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mla, "_lib", None)
    monkeypatch.setattr(mla, "LIB_PATH", str(tmp_path / "libmla.so"))
    with pytest.raises(mla.MlaError):
        mla.lib()


def _noalloc(d, **kw):
    a = dict(q=FAKE, cache=FAKE, npages=100000, table=FAKE, maxp=4, lens=FAKE, batch=2, qlen=1,
             maxlen=256, causal=1, err=FAKE, o=FAKE, lse=FAKE)
    a.update(kw)
    return mla.lib().mla_decode_attn_noalloc(ctypes.byref(d), a["q"], a["cache"], a["npages"],
                                             a["table"], a["maxp"], a["lens"], a["batch"],
                                             a["qlen"], a["maxlen"], a["causal"], a["err"],
                                             a["o"], a["lse"], None)


def test_noalloc_validation_before_launch(mla_lib):
    """The no-allocation decode validates exactly like mla_decode_attn, batch 0 included,
    and refuses a plan larger than its scratch array before any launch or CUDA call."""
    assert _noalloc(_dims(), err=None) == mla.MLA_ERR_INVALID_ARG      # error word required
    assert _noalloc(_dims(page_size=32), batch=0) == mla.MLA_ERR_UNSUPPORTED
    assert _noalloc(_dims(), batch=0, causal=2) == mla.MLA_ERR_INVALID_ARG
    assert _noalloc(_dims(), batch=0, qlen=0) == mla.MLA_ERR_INVALID_ARG
    assert _noalloc(_dims(), batch=0) == mla.MLA_OK                     # valid, nothing to do
    # four million one-page sequences: the per-sequence schedule alone is 16 MB and the
    # automatic plan (the smallest one) no longer fits the 32 MiB array
    d = _dims()
    assert mla.mla_decode_workspace_size(d, 4_000_000, 1, 64, 0) > 32 << 20
    assert _noalloc(d, batch=4_000_000, maxlen=64, maxp=1) == mla.MLA_ERR_WORKSPACE


def test_kv_shared_validation(mla_lib):
    L = mla.lib()
    kv = _dims(CONFIGS["nanowhale_kv_shared"])
    out = mla.MlaDims()
    assert L.mla_kv_shared_decode_dims(ctypes.byref(kv), ctypes.byref(out)) == mla.MLA_OK
    assert (out.kv_lora_rank, out.rope_dim, out.v_head_dim, out.num_kv_groups) == (512, 0, 512, 1)
    assert mla.mla_row_width(out) == 512
    # not a K = V layout: two key groups, d_n != r, d_v != D, no rotary dims
    for bad in (dict(num_kv_groups=2), dict(qk_nope_dim=128), dict(v_head_dim=448),
                dict(rope_dim=0, v_head_dim=448)):
        d = _dims(CONFIGS["nanowhale_kv_shared"], **bad)
        assert L.mla_kv_shared_decode_dims(ctypes.byref(d), ctypes.byref(out)) == \
            mla.MLA_ERR_INVALID_ARG, bad
        assert L.mla_kv_shared_query(ctypes.byref(d), FAKE, FAKE, FAKE, 2, 1, FAKE, None) == \
            mla.MLA_ERR_INVALID_ARG, bad
    assert L.mla_kv_shared_query(ctypes.byref(kv), None, FAKE, FAKE, 2, 1, FAKE, None) == \
        mla.MLA_ERR_INVALID_ARG
    assert L.mla_kv_shared_output(ctypes.byref(kv), FAKE, FAKE, FAKE, 2, 1, P(0x10008), None) == \
        mla.MLA_ERR_INVALID_ARG                                   # misaligned output
    assert L.mla_kv_shared_output(ctypes.byref(kv), FAKE, FAKE, FAKE, 2, 0, FAKE, None) == \
        mla.MLA_ERR_INVALID_ARG                                   # q_len 0
    assert L.mla_kv_shared_query(ctypes.byref(kv), FAKE, FAKE, FAKE, 0, 1, FAKE, None) == mla.MLA_OK


def test_down_kv_append_validation(mla_lib):
    L = mla.lib()
    d = _dims()

    def call(dd=d, hidden=FAKE, hid=5120, w=FAKE, batch=2, n=1, cache=FAKE, kv_out=None):
        return L.mla_down_kv_append(ctypes.byref(dd), hidden, hid, w, FAKE, FAKE, FAKE, 4, FAKE,
                                    batch, n, cache, 100, None, kv_out, None)
    assert call(hid=100) == mla.MLA_ERR_INVALID_ARG              # not a multiple of 8
    assert call(hidden=None) == mla.MLA_ERR_INVALID_ARG
    assert call(w=P(0x10008)) == mla.MLA_ERR_INVALID_ARG          # misaligned weight
    assert call(kv_out=P(0x10004)) == mla.MLA_ERR_INVALID_ARG     # misaligned kv_out
    assert call(dd=_dims(num_kv_groups=4, num_heads=128, rope_dim=64)) == mla.MLA_ERR_UNSUPPORTED
    assert call(batch=0) == mla.MLA_OK
    assert call(n=0) == mla.MLA_OK


def test_out_proj_validation(mla_lib):
    L = mla.lib()
    d = _dims()
    assert mla.mla_out_proj_workspace_size(d, 5120, 64) > 0
    assert mla.mla_out_proj_workspace_size(d, 5121, 64) == 0             # hidden % 8
    assert mla.mla_out_proj_workspace_size(_dims(v_head_dim=96), 5120, 64) == 0   # d_v % 64

    def call(dd=d, ol=FAKE, wo=FAKE, hidden=5120, rows=4, ws=P(0x10000), wsb=1 << 30, u=FAKE):
        return L.mla_out_proj(ctypes.byref(dd), ol, FAKE, 128 * 512, None, wo, None, hidden, rows,
                              ws, wsb, FAKE, u, None)
    assert call(ol=None) == mla.MLA_ERR_INVALID_ARG
    assert call(u=P(0x10002)) == mla.MLA_ERR_INVALID_ARG
    assert call(ws=None) == mla.MLA_ERR_WORKSPACE
    assert call(wsb=64) == mla.MLA_ERR_WORKSPACE
    assert call(dd=_dims(v_head_dim=96)) == mla.MLA_ERR_UNSUPPORTED
    assert call(rows=0) == mla.MLA_OK
