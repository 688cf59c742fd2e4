"""CPU fp64 oracle for weight-absorbed MLA decode.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The product (the CUDA library and its
Python binding) never calls it and shares no code with it.

What it computes, and where the pages define it
------------------------------------------------
* ``mla_decode_reference``: attention in the UNABSORBED form. Every cached latent
  c_kv[l] is up-projected into a full per-head key K_h[l] = [W_UK[h] c_kv[l]; R(l) k_r[l, g(h)]]
  and value V_h[l] = W_UV[h] c_kv[l] (+ bias_h); the query is Q = [q_nope; R(pos) q_pe];
  then ordinary softmax attention (DeepSeek-V2 MLA page, dtcms.com: "compute attention
  after up-projection" and the original-order einsums (1)-(3) of the "Matrix absorption"
  section). The absorbed kernels reach the same result by associativity (einsums (4)-(5)
  of that section), so this plain definition is the reference for them.
  It also returns o_latent = sum_l p_l c_kv[l], the intermediate of einsum (4).
* ``absorb_reference`` / ``out_up_reference``: the absorb einsum and einsum (5) on their
  own, for checking the two projection steps separately.
* ``mla_decode_absorbed``: the same attention in the absorbed order (a second CPU
  baseline; equal to the unabsorbed definition by associativity).
* ``o_proj_reference``: einsum (6), the output projection of the heads' values to the
  model width (W_o of shape [H, d_v, hidden]).
* ``down_kv_reference``: the hidden -> [c_kv ; k_r] projection whose output the cache
  stores (down_kv / k_r_proj of the MLAfication page, kv_a_proj_with_mqa of the
  DeepSeek-V2 page).
* ``kv_shared_reference``: the single-latent K = V form of the nanowhale-100m page
  (cnnetsun.cn): one rotated head_dim vector per token serves as key and value, and the
  output's rotary dims are rotated back by the query position.
* ``rope_rotate``: RoPE on a rotary slice, pairs (x_j, x_{j+d/2}) rotated by theta_j * pos
  (the rotate-half convention of ``apply_rotary_pos_emb`` used on that page), angles in fp64.
* ``cache_append_emulate``: the byte-exact result of writing new tokens into the paged
  latent cache. The cache row holds the latent c_kv followed by each group's rotated
  key (the "cache stores only c_kv" data flow of the MLAfication page, wzjinhao.cn, and
  the ``torch.split(compressed_kv, [kv_lora_rank, qk_rope_head_dim])`` row layout of the
  DeepSeek-V2 page). The rotation is emulated in fp32 with separately rounded multiply,
  subtract and add, from the same fp32 cos/sin tables the GPU receives, then rounded
  to bf16 (round to nearest, ties to even).

Readings where the pages are silent: softmax is plain (no dropout, sink or bias); the
causal mask lets query row i see token l iff l <= its position; lse is the natural log;
head h uses key group g(h) = h // (H / G).

Memory is bounded by looping over heads and over chunks of the context when building
the scores; each score is still one independent dot product, and the softmax and the
weighted sums run over the whole context, so nothing is reordered beyond the
order of fp64 summation.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

_CHUNK = 1 << 16


def as_f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or numpy array -> float64 numpy (exact for bf16/fp32)."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def group_of_head(num_heads: int, num_groups: int) -> np.ndarray:
    return np.arange(num_heads) // (num_heads // num_groups)


def rope_rotate(x: np.ndarray, theta: np.ndarray, pos) -> np.ndarray:
    """Rotate pairs (x_j, x_{j+d/2}) of x[..., d] by angle theta_j * pos (fp64).

    ``pos`` broadcasts against ``x[..., 0]``.
    """
    d = x.shape[-1]
    h = d // 2
    if d == 0:
        return x.copy()
    ang = np.asarray(pos, dtype=np.float64)[..., None] * np.asarray(theta, dtype=np.float64)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., :h], x[..., h:]
    return np.concatenate([x0 * c - x1 * s, x1 * c + x0 * s], axis=-1)


def mla_decode_reference(q_nope, q_pe, c_kv, k_r, w_uk, w_uv, bias, theta, q_pos,
                         softmax_scale: float, causal: bool = True,
                         want_p: bool = False) -> Dict[str, np.ndarray]:
    """Unabsorbed MLA attention for ONE sequence, in fp64.

    q_nope [q, H, d_n], q_pe [q, H, d_r] (unrotated), c_kv [L, r], k_r [L, G, d_r]
    (unrotated; token l sits at position l), w_uk [H, d_n, r], w_uv [H, d_v, r],
    bias [H, d_v] or None, theta [G, d_r/2], q_pos [q] (query positions).
    Returns o [q, H, d_v], o_latent [q, H, r], lse [q, H] and, if asked, p [q, H, L].
    """
    q_nope, q_pe, c_kv, k_r = as_f64(q_nope), as_f64(q_pe), as_f64(c_kv), as_f64(k_r)
    w_uk, w_uv = as_f64(w_uk), as_f64(w_uv)
    bias = None if bias is None else as_f64(bias)
    theta = np.asarray(theta, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    nq, H, _ = q_nope.shape
    L, r = c_kv.shape
    G = k_r.shape[1]
    dv = w_uv.shape[1]
    g_of = group_of_head(H, G)
    tok_pos = np.arange(L, dtype=np.int64)

    # RoPE: keys at their own positions, queries at theirs.
    k_rot = np.empty_like(k_r)
    for g in range(G):
        k_rot[:, g, :] = rope_rotate(k_r[:, g, :], theta[g], tok_pos)
    q_rot = np.empty_like(q_pe)
    for h in range(H):
        q_rot[:, h, :] = rope_rotate(q_pe[:, h, :], theta[g_of[h]], q_pos)

    visible = np.ones((nq, L), dtype=bool)
    if causal:
        visible = tok_pos[None, :] <= q_pos[:, None]

    o = np.zeros((nq, H, dv))
    o_lat = np.zeros((nq, H, r))
    lse = np.zeros((nq, H))
    p_all = np.zeros((nq, H, L)) if want_p else None
    for h in range(H):
        Q = np.concatenate([q_nope[:, h, :], q_rot[:, h, :]], axis=-1)        # [q, d_n + d_r]
        s = np.empty((nq, L))
        for l0 in range(0, L, _CHUNK):
            l1 = min(L, l0 + _CHUNK)
            K_nope = c_kv[l0:l1] @ w_uk[h].T                                  # [l, d_n] = W_UK[h] c_kv[l]
            K = np.concatenate([K_nope, k_rot[l0:l1, g_of[h], :]], axis=-1)  # [l, d_n + d_r]
            s[:, l0:l1] = softmax_scale * (Q @ K.T)
        s = np.where(visible, s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        lse_h = m[:, 0] + np.log(np.exp(s - m).sum(axis=-1))
        p = np.exp(s - lse_h[:, None])                                       # rows sum to 1
        lse[:, h] = lse_h
        acc_v = np.zeros((nq, dv))
        acc_c = np.zeros((nq, r))
        for l0 in range(0, L, _CHUNK):
            l1 = min(L, l0 + _CHUNK)
            V = c_kv[l0:l1] @ w_uv[h].T                                       # [l, d_v] = W_UV[h] c_kv[l]
            if bias is not None:
                V = V + bias[h]
            acc_v += p[:, l0:l1] @ V
            acc_c += p[:, l0:l1] @ c_kv[l0:l1]
        o[:, h, :] = acc_v
        o_lat[:, h, :] = acc_c
        if want_p:
            p_all[:, h, :] = p
    out = {"o": o, "o_latent": o_lat, "lse": lse}
    if want_p:
        out["p"] = p_all
    return out


def absorb_reference(q_nope, q_pe, w_uk, theta, q_pos, num_groups: int):
    """Absorb step in fp64: q_c = einsum('hdc,ihd->ihc', W_UK, q_nope) (the q_absorb einsum
    of the "Matrix absorption" listing) and the rotated q_pe of each head at its row's
    position. q_nope [q, H, d_n], q_pe [q, H, d_r] -> (q_c [q, H, r], q_rot [q, H, d_r])."""
    q_nope, q_pe, w_uk = as_f64(q_nope), as_f64(q_pe), as_f64(w_uk)
    H = w_uk.shape[0]
    g_of = group_of_head(H, num_groups)
    q_c = np.einsum("hdc,ihd->ihc", w_uk, q_nope)
    q_rot = np.empty_like(q_pe)
    for h in range(H):
        q_rot[:, h, :] = rope_rotate(q_pe[:, h, :], np.asarray(theta)[g_of[h]], np.asarray(q_pos))
    return q_c, q_rot


def out_up_reference(o_latent, w_uv, bias=None):
    """Einsum (5) of the "Matrix absorption" section, o = einsum('ihc,hdc->ihd', o_, W_UV),
    plus the optional up_v bias. o_latent [..., H, r] -> [..., H, d_v]."""
    o = np.einsum("...hc,hdc->...hd", as_f64(o_latent), as_f64(w_uv))
    if bias is not None:
        o = o + as_f64(bias)
    return o


# ----------------------------------------------------------------------------------------
# Byte-level emulation of the cache append
# ----------------------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest with ties to even; NaN -> 0x7FC0."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    return np.where(nan, np.uint16(0x7FC0), rounded).astype(np.uint16)


def rotate_fp32(x: np.ndarray, cos32: np.ndarray, sin32: np.ndarray) -> np.ndarray:
    """fp32 rotation of pairs (x_j, x_{j+d/2}) with every product and sum rounded to fp32."""
    h = x.shape[-1] // 2
    x0 = x[..., :h].astype(np.float32)
    x1 = x[..., h:].astype(np.float32)
    c = cos32.astype(np.float32)
    s = sin32.astype(np.float32)
    y0 = np.subtract(np.multiply(x0, c, dtype=np.float32), np.multiply(x1, s, dtype=np.float32),
                     dtype=np.float32)
    y1 = np.add(np.multiply(x1, c, dtype=np.float32), np.multiply(x0, s, dtype=np.float32),
                dtype=np.float32)
    return np.concatenate([y0, y1], axis=-1)


def cache_append_emulate(cache_bits: np.ndarray, c_kv_bits: np.ndarray, k_r_bits: np.ndarray,
                         cos32: np.ndarray, sin32: np.ndarray, block_table: np.ndarray,
                         start_pos: np.ndarray, page_size: int) -> np.ndarray:
    """Return a copy of ``cache_bits`` [num_pages, page_size, D] (uint16) after appending.

    c_kv_bits [B, n, r], k_r_bits [B, n, G, d_r] (uint16 bf16 patterns), cos32/sin32
    [B, n, G, d_r/2] fp32, block_table [B, max_pages] int32, start_pos [B].
    Token t of sequence b lands at position p = start_pos[b] + t, i.e. in physical page
    block_table[b, p // page_size], row p % page_size.
    """
    out = np.array(cache_bits, dtype=np.uint16, copy=True)
    B, n, r = c_kv_bits.shape
    G, dr = k_r_bits.shape[2], k_r_bits.shape[3]
    for b in range(B):
        pos = int(start_pos[b]) + np.arange(n)
        pages = block_table[b, pos // page_size].astype(np.int64)
        rows = pos % page_size
        out[pages, rows, :r] = c_kv_bits[b]
        if dr > 0:
            x = bf16_bits_to_f32(k_r_bits[b])                              # [n, G, d_r]
            y = rotate_fp32(x, cos32[b], sin32[b])                         # [n, G, d_r]
            out[pages, rows, r:] = f32_to_bf16_bits(y).reshape(n, G * dr)
    return out


# ----------------------------------------------------------------------------------------
# The single-latent K = V form (nanowhale-100m page, cnnetsun.cn)
# ----------------------------------------------------------------------------------------

def kv_shared_reference(q_nope, q_pe, kv_nope, kv_pe, theta, q_pos, softmax_scale,
                        causal: bool = True) -> Dict[str, np.ndarray]:
    """Attention in which one cached vector per token is both key and value, in fp64.

    The nanowhale-100m page ("single KV head, many query heads"; "applying RoPE"; "efficient
    attention": scaled_dot_product_attention(q, kv_expanded, kv_expanded)): every head's
    query attends over one shared head_dim vector per token, kv = [kv_nope ; kv_pe], whose
    last d_r dims are rotated at the token's position, as are the query's last d_r dims at
    the query position; the values are the same rotated vectors, so the output's last d_r
    dims are a mix of vectors rotated to different positions. The page's "output inverse
    rotation" then rotates those dims back by the query's own position (reading: the
    position of the output row).

    q_nope [q, H, d_n], q_pe [q, H, d_r] (unrotated), kv_nope [L, d_n], kv_pe [L, d_r]
    (unrotated; token l at position l), theta [d_r/2], q_pos [q].
    Returns o [q, H, d_n + d_r] (after the inverse rotation) and lse [q, H].
    """
    q_nope, q_pe = as_f64(q_nope), as_f64(q_pe)
    kv_nope, kv_pe = as_f64(kv_nope), as_f64(kv_pe)
    theta = np.asarray(theta, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    nq, H, _ = q_nope.shape
    L = kv_nope.shape[0]
    tok_pos = np.arange(L, dtype=np.int64)
    kv = np.concatenate([kv_nope, rope_rotate(kv_pe, theta, tok_pos)], axis=-1)       # [L, Dh]
    q_rot = rope_rotate(q_pe, theta, q_pos[:, None])                                   # [q, H, d_r]
    Q = np.concatenate([q_nope, q_rot], axis=-1)                                       # [q, H, Dh]
    s = softmax_scale * np.einsum("ihd,ld->ihl", Q, kv)
    if causal:
        s = np.where((tok_pos[None, :] <= q_pos[:, None])[:, None, :], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    lse = m[..., 0] + np.log(np.exp(s - m).sum(axis=-1))
    p = np.exp(s - lse[..., None])
    o = np.einsum("ihl,ld->ihd", p, kv)                                                # V = K
    dn = kv_nope.shape[1]
    o[..., dn:] = rope_rotate(o[..., dn:], theta, -q_pos[:, None])                     # inverse
    return {"o": o, "lse": lse}


def mla_decode_absorbed(q_nope, q_pe, c_kv, k_r, w_uk, w_uv, bias, theta, q_pos,
                        softmax_scale: float, causal: bool = True) -> Dict[str, np.ndarray]:
    """The same attention in the absorbed order, in fp64, for ONE sequence: q_c =
    einsum('hdc,bhqd->bhqc', W_UK, q_nope), scores q_c . c_kv + rotated q_pe . rotated k_r,
    o_ = p c_kv (einsum 4), o = o_ W_UV (einsum 5) (DeepSeek-V2 page, "Matrix absorption").
    Arguments and results as mla_decode_reference. Used as a second CPU baseline; it equals
    the unabsorbed definition by associativity."""
    q_nope, q_pe, c_kv, k_r = as_f64(q_nope), as_f64(q_pe), as_f64(c_kv), as_f64(k_r)
    w_uk, w_uv = as_f64(w_uk), as_f64(w_uv)
    theta = np.asarray(theta, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    nq, H, _ = q_nope.shape
    L = c_kv.shape[0]
    G = k_r.shape[1]
    g_of = group_of_head(H, G)
    tok_pos = np.arange(L, dtype=np.int64)
    q_c, q_rot = absorb_reference(q_nope, q_pe, w_uk, theta, q_pos, G)
    o_lat = np.zeros((nq, H, c_kv.shape[1]))
    lse = np.zeros((nq, H))
    for g in range(G):
        k_rot = rope_rotate(k_r[:, g, :], theta[g], tok_pos)                           # [L, d_r]
        hs = np.nonzero(g_of == g)[0]
        s = softmax_scale * (np.einsum("ihc,lc->ihl", q_c[:, hs], c_kv) +
                             np.einsum("ihe,le->ihl", q_rot[:, hs], k_rot))
        if causal:
            s = np.where((tok_pos[None, :] <= q_pos[:, None])[:, None, :], s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        lse_g = m[..., 0] + np.log(np.exp(s - m).sum(axis=-1))
        o_lat[:, hs] = np.einsum("ihl,lc->ihc", np.exp(s - lse_g[..., None]), c_kv)    # (4)
        lse[:, hs] = lse_g
    o = out_up_reference(o_lat, w_uv, None if bias is None else as_f64(bias))          # (5)
    return {"o": o, "o_latent": o_lat, "lse": lse}


# ----------------------------------------------------------------------------------------
# The KV down-projection that produces the cached latent (fused with the append on the GPU)
# ----------------------------------------------------------------------------------------

def down_kv_reference(hidden, w_dkv, kv_lora_rank: int, num_groups: int, rope_dim: int):
    """The cached token's latent and unrotated rotary key from its hidden state, in fp64.

    The MLAfication page (wzjinhao.cn) sends the hidden state X through down_kv to the
    latent c_kv (the only part of K/V the cache keeps) and through k_r_proj to the low-
    dimensional rotary key; the DeepSeek-V2 page does both with one matrix, eq. (41)
    kv_a_proj_with_mqa, whose output is split into [kv_lora_rank, qk_rope_head_dim]. Here
    w_dkv [r + G*d_r, hidden] stacks the down_kv rows and each group's k_r rows, and
    [c_kv ; k_r] = w_dkv @ x for every token x [.., hidden].
    Returns c_kv [.., r] and k_r [.., G, d_r] (fp64, before RoPE).
    """
    out = np.einsum("...k,dk->...d", as_f64(hidden), as_f64(w_dkv))
    c_kv = out[..., :kv_lora_rank]
    k_r = out[..., kv_lora_rank:].reshape(out.shape[:-1] + (num_groups, rope_dim))
    return c_kv, k_r


def o_proj_reference(o, w_o, bias=None):
    """The output projection, einsum (6) of the "Matrix absorption" section:
    u = einsum('hdD,bhqd->bqD', W_o, o), i.e. u[.., D] = sum over heads h and value dims d of
    W_o[h, d, D] o[.., h, d] (+ bias[D]). o [..., H, d_v], w_o [H, d_v, hidden] -> [..., hidden]."""
    u = np.einsum("...hd,hdk->...k", as_f64(o), as_f64(w_o))
    if bias is not None:
        u = u + as_f64(bias)
    return u
