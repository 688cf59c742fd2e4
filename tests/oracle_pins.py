"""Pins that tie the CPU oracle to facts outside itself.

Each ``pin_*`` takes the oracle module and raises AssertionError on failure, so the
same checks run against the real oracle (tests/test_oracle_pins.py) and against
copies of it with a planted mistake (tests/test_oracle_mutations.py).

What pins what:
* brute force: literal scalar loops over (query row, head, token) written from the
  definition of attention with up-projected keys/values (DeepSeek-V2 MLA page,
  "compute attention after up-projection"), tiny shapes, G > 1, causal q > 1, bias.
* associativity: the absorbed order of the "Matrix absorption" section (q_c from
  einsum 'hdc,bhqd->bhqc', scores on the compressed cache, einsum (4) then (5)) equals
  the oracle's unabsorbed order (einsums (1)-(3)).
* library routine: with identity up-projections and no rotary part the method is
  multi-query attention over c_kv; torch's scaled_dot_product_attention (fp64, CPU)
  computes it independently.
* closed forms: q = 0 gives uniform weights (lse = ln of the visible count, o = mean
  value); L = 1 gives o = V_0 and o_latent = c_0; softmax rows sum to one.
* RoPE: rotation matches complex multiplication by exp(i theta pos), keeps norms,
  and the rotated dot product depends only on the position difference.
* cache append: bf16 rounding equals torch's float32 -> bfloat16 conversion; slot
  addressing equals a per-token dictionary write; the fp32 rotation stays within
  fp32 rounding of the fp64 rotation.
"""
from __future__ import annotations

import math

import numpy as np
import torch


# ----------------------------------------------------------------------------------------
# small random problems
# ----------------------------------------------------------------------------------------

def _problem(seed, nq=2, H=4, G=2, r=3, dn=2, dr=4, dv=2, L=6, bias=True, scale=0.7):
    rng = np.random.default_rng(seed)
    P = dict(
        q_nope=rng.standard_normal((nq, H, dn)),
        q_pe=rng.standard_normal((nq, H, dr)),
        c_kv=rng.standard_normal((L, r)),
        k_r=rng.standard_normal((L, G, dr)),
        w_uk=rng.standard_normal((H, dn, r)),
        w_uv=rng.standard_normal((H, dv, r)),
        bias=rng.standard_normal((H, dv)) if bias else None,
        theta=rng.uniform(0.05, 1.3, size=(G, dr // 2)),
        q_pos=np.arange(L - nq, L),
        softmax_scale=scale,
    )
    return P


def _brute_force(q_nope, q_pe, c_kv, k_r, w_uk, w_uv, bias, theta, q_pos, softmax_scale,
                 causal=True):
    nq, H, dn = q_nope.shape
    L, r = c_kv.shape
    G, dr = k_r.shape[1], k_r.shape[2]
    dv = w_uv.shape[1]
    half = dr // 2
    hpg = H // G
    o = np.zeros((nq, H, dv))
    o_lat = np.zeros((nq, H, r))
    lse = np.zeros((nq, H))
    for i in range(nq):
        for h in range(H):
            g = h // hpg
            qr = [0.0] * dr
            for j in range(half):
                a = theta[g][j] * q_pos[i]
                x0, x1 = q_pe[i][h][j], q_pe[i][h][j + half]
                qr[j] = x0 * math.cos(a) - x1 * math.sin(a)
                qr[j + half] = x1 * math.cos(a) + x0 * math.sin(a)
            scores = []
            for l in range(L):
                if causal and l > q_pos[i]:
                    scores.append(None)
                    continue
                sc = 0.0
                for d in range(dn):
                    kd = 0.0
                    for c in range(r):
                        kd += w_uk[h][d][c] * c_kv[l][c]
                    sc += q_nope[i][h][d] * kd
                for j in range(half):
                    a = theta[g][j] * l
                    x0, x1 = k_r[l][g][j], k_r[l][g][j + half]
                    k0 = x0 * math.cos(a) - x1 * math.sin(a)
                    k1 = x1 * math.cos(a) + x0 * math.sin(a)
                    sc += qr[j] * k0 + qr[j + half] * k1
                scores.append(softmax_scale * sc)
            mx = max(s for s in scores if s is not None)
            z = sum(math.exp(s - mx) for s in scores if s is not None)
            lse[i][h] = mx + math.log(z)
            p = [0.0 if s is None else math.exp(s - lse[i][h]) for s in scores]
            for d in range(dv):
                acc = 0.0
                for l in range(L):
                    v = 0.0
                    for c in range(r):
                        v += w_uv[h][d][c] * c_kv[l][c]
                    if bias is not None:
                        v += bias[h][d]
                    acc += p[l] * v
                o[i][h][d] = acc
            for c in range(r):
                o_lat[i][h][c] = sum(p[l] * c_kv[l][c] for l in range(L))
    return {"o": o, "o_latent": o_lat, "lse": lse}


def _close(a, b, rtol, what):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    ref = max(np.max(np.abs(b)) if b.size else 0.0, 1e-300)
    assert err <= rtol * ref, f"{what}: max|err| {err:.3e} > {rtol:.1e} * {ref:.3e}"


# ----------------------------------------------------------------------------------------
# pins on the decode reference
# ----------------------------------------------------------------------------------------

def pin_bruteforce(O):
    for seed, kw in [(1, {}), (2, dict(nq=1, H=2, G=1, r=4, dn=3, dr=2, dv=3, L=5)),
                     (3, dict(nq=3, H=6, G=3, r=2, dn=2, dr=2, dv=1, L=4, bias=False)),
                     (4, dict(nq=2, H=4, G=2, r=4, dn=4, dr=6, dv=4, L=3))]:
        P = _problem(seed, **kw)
        ref = _brute_force(**P)
        got = O.mla_decode_reference(**P)
        for k in ("o", "o_latent", "lse"):
            _close(got[k], ref[k], 1e-11, f"bruteforce seed {seed} {k}")


def _absorbed(O, q_nope, q_pe, c_kv, k_r, w_uk, w_uv, bias, theta, q_pos, softmax_scale):
    """Absorbed order: q_c = einsum('hdc,ihd->ihc'), scores on (c_kv, rotated k_r),
    o_ = p c_kv (einsum 4), o = einsum('ihc,hdc->ihd', o_, W_UV) (einsum 5)."""
    nq, H, _ = q_nope.shape
    L = c_kv.shape[0]
    G = k_r.shape[1]
    g_of = np.arange(H) // (H // G)
    k_rot = np.stack([O.rope_rotate(k_r[:, g, :], theta[g], np.arange(L)) for g in range(G)], 1)
    q_rot = np.stack([O.rope_rotate(q_pe[:, h, :], theta[g_of[h]], q_pos) for h in range(H)], 1)
    q_c = np.einsum("hdc,ihd->ihc", w_uk, q_nope)
    s = np.einsum("ihc,lc->ihl", q_c, c_kv) + np.einsum("ihe,lhe->ihl", q_rot, k_rot[:, g_of, :])
    s = s * softmax_scale
    vis = np.arange(L)[None, :] <= np.asarray(q_pos)[:, None]
    s = np.where(vis[:, None, :], s, -np.inf)
    m = s.max(-1, keepdims=True)
    e = np.exp(s - m)
    p = e / e.sum(-1, keepdims=True)
    o_ = np.einsum("ihl,lc->ihc", p, c_kv)
    o = np.einsum("ihc,hdc->ihd", o_, w_uv)
    if bias is not None:
        o = o + bias[None]
    return o, o_


def pin_associativity(O):
    for seed, kw in [(11, dict(nq=1, H=8, G=1, r=16, dn=8, dr=8, dv=8, L=40)),
                     (12, dict(nq=4, H=8, G=4, r=12, dn=6, dr=4, dv=5, L=33)),
                     (13, dict(nq=2, H=6, G=2, r=8, dn=8, dr=2, dv=8, L=17, bias=False))]:
        P = _problem(seed, **kw)
        got = O.mla_decode_reference(**P)
        o, o_ = _absorbed(O, **P)
        _close(got["o"], o, 1e-11, "absorbed o")
        _close(got["o_latent"], o_, 1e-11, "absorbed o_latent")


def pin_sdpa_identity_weights(O):
    """d_n = d_v = r, W_UK = W_UV = I, no rotary dims: MQA over c_kv, checked with SDPA."""
    rng = np.random.default_rng(21)
    nq, H, r, L = 3, 5, 8, 29
    qn = rng.standard_normal((nq, H, r))
    c_kv = rng.standard_normal((L, r))
    eye = np.broadcast_to(np.eye(r), (H, r, r)).copy()
    scale = 0.43
    q_pos = np.arange(L - nq, L)
    got = O.mla_decode_reference(qn, np.zeros((nq, H, 0)), c_kv, np.zeros((L, 1, 0)), eye, eye,
                                 None, np.zeros((1, 0)), q_pos, scale, causal=True)
    q = torch.from_numpy(qn).permute(1, 0, 2)[None]                         # [1, H, q, r]
    kv = torch.from_numpy(c_kv)[None, None].expand(1, H, L, r)
    mask = torch.from_numpy(np.arange(L)[None, :] <= q_pos[:, None])
    ref = torch.nn.functional.scaled_dot_product_attention(q, kv, kv, attn_mask=mask, scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    _close(got["o"], ref, 1e-12, "sdpa o")
    _close(got["o_latent"], ref, 1e-12, "sdpa o_latent")
    s = np.einsum("ihc,lc->ihl", qn, c_kv) * scale
    s = np.where(mask.numpy()[:, None, :], s, -np.inf)
    lse_ref = torch.logsumexp(torch.from_numpy(s), dim=-1).numpy()
    _close(got["lse"], lse_ref, 1e-12, "sdpa lse")


def pin_zero_query_uniform(O):
    P = _problem(31, nq=3, H=4, G=2, r=5, dn=3, dr=4, dv=3, L=9)
    P["q_nope"] = np.zeros_like(P["q_nope"])
    P["q_pe"] = np.zeros_like(P["q_pe"])
    got = O.mla_decode_reference(**P)
    L = P["c_kv"].shape[0]
    for i, qp in enumerate(P["q_pos"]):
        n_vis = qp + 1
        assert np.allclose(got["lse"][i], math.log(n_vis), rtol=0, atol=1e-13), "uniform lse"
        mean_c = P["c_kv"][:n_vis].mean(0)
        _close(got["o_latent"][i], np.broadcast_to(mean_c, got["o_latent"][i].shape), 1e-12,
               "uniform o_latent")
        mean_v = np.einsum("hdc,c->hd", P["w_uv"], mean_c) + P["bias"]
        _close(got["o"][i], mean_v, 1e-12, "uniform o")
    assert L == 9


def pin_single_token(O):
    P = _problem(41, nq=1, H=3, G=1, r=4, dn=2, dr=2, dv=3, L=1)
    P["q_pos"] = np.array([0])
    got = O.mla_decode_reference(**P)
    v0 = np.einsum("hdc,c->hd", P["w_uv"], P["c_kv"][0]) + P["bias"]
    _close(got["o"][0], v0, 1e-13, "L=1 o")
    _close(got["o_latent"][0], np.broadcast_to(P["c_kv"][0], (3, 4)), 1e-13, "L=1 o_latent")


def pin_rows_sum_to_one(O):
    P = _problem(51, nq=4, H=4, G=2, r=6, dn=4, dr=4, dv=4, L=23)
    got = O.mla_decode_reference(**P, want_p=True)
    p = got["p"]
    assert np.all(p >= 0)
    assert np.allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14), "rows sum to 1"
    L = P["c_kv"].shape[0]
    for i, qp in enumerate(P["q_pos"]):
        assert np.all(p[i, :, qp + 1:] == 0.0), "masked weights are zero"
    assert p.shape[-1] == L


def pin_causal_prefix(O):
    """Row i of a causal q-block equals a single-query call on its visible prefix."""
    P = _problem(61, nq=4, H=4, G=2, r=5, dn=3, dr=4, dv=2, L=12)
    got = O.mla_decode_reference(**P)
    for i, qp in enumerate(P["q_pos"]):
        sub = dict(P)
        sub["q_nope"] = P["q_nope"][i:i + 1]
        sub["q_pe"] = P["q_pe"][i:i + 1]
        sub["c_kv"] = P["c_kv"][:qp + 1]
        sub["k_r"] = P["k_r"][:qp + 1]
        sub["q_pos"] = np.array([qp])
        one = O.mla_decode_reference(**sub)
        for k in ("o", "o_latent", "lse"):
            _close(got[k][i], one[k][0], 1e-12, f"causal prefix {k}")


# ----------------------------------------------------------------------------------------
# RoPE pins
# ----------------------------------------------------------------------------------------

def pin_rope_complex(O):
    rng = np.random.default_rng(71)
    x = rng.standard_normal((50, 8))
    theta = rng.uniform(0.01, 2.0, size=4)
    pos = rng.integers(0, 100000, size=50)
    y = O.rope_rotate(x, theta, pos)
    z = (x[:, :4] + 1j * x[:, 4:]) * np.exp(1j * theta[None, :] * pos[:, None])
    _close(y, np.concatenate([z.real, z.imag], -1), 1e-12, "rope vs complex")


def pin_rope_norm_and_relative(O):
    rng = np.random.default_rng(72)
    q = rng.standard_normal(16)
    k = rng.standard_normal(16)
    theta = 10000.0 ** (-np.arange(8) / 8.0)
    assert abs(np.linalg.norm(O.rope_rotate(q, theta, 12345)) - np.linalg.norm(q)) < 1e-12
    d1 = O.rope_rotate(q, theta, 17) @ O.rope_rotate(k, theta, 5)
    d2 = O.rope_rotate(q, theta, 112) @ O.rope_rotate(k, theta, 100)
    assert abs(d1 - d2) < 1e-11, "relative-position property"
    assert np.array_equal(O.rope_rotate(q, np.zeros(8), 77), q), "zero angle is identity"


# ----------------------------------------------------------------------------------------
# cache-append emulation pins
# ----------------------------------------------------------------------------------------

def pin_bf16_rounding(O):
    rng = np.random.default_rng(81)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        np.array([0.0, -0.0, 1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8),
                  3.4028235e38, 3.39e38, 1e-40, -1e-42, np.inf, -np.inf, 2.0 ** -126,
                  65504.0, 1.00390625, 1.01171875], dtype=np.float32),
        (rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
         .view(np.float32)),
    ]).astype(np.float32)
    x = x[~np.isnan(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f32_to_bf16_bits(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"bf16 rounding differs at {x[bad[:5]]}: {got[bad[:5]]} vs {ref[bad[:5]]}"
    nan = O.f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))
    assert (int(nan[0]) & 0x7F80) == 0x7F80 and (int(nan[0]) & 0x7F) != 0, "NaN stays NaN"
    bits = rng.integers(0, 2 ** 16, size=5000).astype(np.uint16)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    f = O.bf16_bits_to_f32(bits)
    ok = np.isnan(back) == np.isnan(f)
    assert ok.all() and np.array_equal(f[~np.isnan(f)], back[~np.isnan(back)]), "bf16 -> f32"


def pin_rotate_fp32(O):
    rng = np.random.default_rng(82)
    x = rng.standard_normal((400, 3, 8)).astype(np.float32)
    ang = rng.uniform(-50, 50, size=(400, 3, 4))
    c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    y = O.rotate_fp32(x, c, s)
    xd, cd, sd = x.astype(np.float64), c.astype(np.float64), s.astype(np.float64)
    ref = np.concatenate([xd[..., :4] * cd - xd[..., 4:] * sd, xd[..., 4:] * cd + xd[..., :4] * sd], -1)
    tol = 4 * np.finfo(np.float32).eps * (np.abs(xd[..., :4]) + np.abs(xd[..., 4:])).max()
    assert np.max(np.abs(y - ref)) <= tol, "fp32 rotation within rounding of fp64"
    ident = O.rotate_fp32(x, np.ones_like(c), np.zeros_like(s))
    assert np.array_equal(ident, x), "cos 1 sin 0 is the identity"
    swap = O.rotate_fp32(x, np.zeros_like(c), np.ones_like(s))
    assert np.array_equal(swap, np.concatenate([-x[..., 4:], x[..., :4]], -1)), "quarter turn"


def pin_append_slots(O):
    rng = np.random.default_rng(91)
    B, n, r, G, dr, ps, npages = 3, 5, 8, 2, 4, 4, 20
    D = r + G * dr
    table = np.full((B, 6), -1, dtype=np.int32)
    perm = rng.permutation(npages)
    start = np.array([0, 3, 9])
    k = 0
    for b in range(B):
        need = (start[b] + n + ps - 1) // ps
        table[b, :need] = perm[k:k + need]
        k += need
    sentinel = np.uint16(0xABCD)
    cache = np.full((npages, ps, D), sentinel, dtype=np.uint16)
    c_bits = rng.integers(0, 2 ** 16, size=(B, n, r)).astype(np.uint16)
    k_f = rng.standard_normal((B, n, G, dr)).astype(np.float32)
    k_bits = torch.from_numpy(k_f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ang = rng.uniform(-3, 3, size=(B, n, G, dr // 2))
    c32, s32 = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    out = O.cache_append_emulate(cache, c_bits, k_bits, c32, s32, table, start, ps)
    written = {}
    for b in range(B):
        for t in range(n):
            p = start[b] + t
            written[(int(table[b, p // ps]), int(p % ps))] = (b, t)
    for pg in range(npages):
        for row in range(ps):
            if (pg, row) not in written:
                assert np.all(out[pg, row] == sentinel), "untouched slot changed"
            else:
                b, t = written[(pg, row)]
                assert np.array_equal(out[pg, row, :r], c_bits[b, t]), "latent copied exactly"
                xk = O.bf16_bits_to_f32(k_bits[b, t]).astype(np.float64)
                for g in range(G):
                    x0, x1 = xk[g, :dr // 2], xk[g, dr // 2:]
                    cc, ss = c32[b, t, g].astype(np.float64), s32[b, t, g].astype(np.float64)
                    want = np.concatenate([x0 * cc - x1 * ss, x1 * cc + x0 * ss])
                    got = O.bf16_bits_to_f32(out[pg, row, r + g * dr: r + (g + 1) * dr])
                    assert np.all(np.abs(got - want) <= 2.0 ** -7 * np.abs(want) + 1e-30), \
                        "rotated key within bf16 rounding"


def pin_absorb_single_token(O):
    """With one cached token lse = s_0; the absorbed score from absorb_reference must equal it."""
    P = _problem(101, nq=2, H=4, G=2, r=6, dn=3, dr=4, dv=2, L=1)
    P["q_pos"] = np.array([0, 0])
    got = O.mla_decode_reference(**P, causal=False)
    q_c, q_rot = O.absorb_reference(P["q_nope"], P["q_pe"], P["w_uk"], P["theta"], P["q_pos"], 2)
    g_of = np.arange(4) // 2
    k_rot = np.stack([O.rope_rotate(P["k_r"][:, g, :], P["theta"][g], np.arange(1)) for g in range(2)], 1)
    s0 = P["softmax_scale"] * (np.einsum("ihc,c->ih", q_c, P["c_kv"][0]) +
                               np.einsum("ihe,he->ih", q_rot, k_rot[0, g_of, :]))
    _close(got["lse"], s0, 1e-12, "absorbed score vs single-token lse")


def pin_out_up_associativity(O):
    """o = W_UV o_latent + bias (einsum 5) equals the unabsorbed o, since weights sum to 1."""
    P = _problem(102, nq=3, H=4, G=1, r=7, dn=3, dr=2, dv=5, L=19)
    got = O.mla_decode_reference(**P)
    _close(O.out_up_reference(got["o_latent"], P["w_uv"], P["bias"]), got["o"], 1e-12, "einsum 5")


# ----------------------------------------------------------------------------------------
# pins on the single-latent K = V form and on the absorbed-order baseline
# ----------------------------------------------------------------------------------------

def _complex_rotate(x, theta, pos):
    """Rotate interleaved pairs (x_2j, x_2j+1) as complex numbers times exp(i theta_j pos)."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * theta)
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def pin_kv_shared_sdpa(O):
    """K = V attention with the page's complex (interleaved-pair) rotary embedding, torch's
    scaled_dot_product_attention with the same tensor as key and value, and the inverse
    rotation of the output by multiplication with exp(-i theta pos_q). The oracle uses
    half-split pairs (x_j, x_j+d/2); the two agree once the rotary dims are permuted."""
    rng = np.random.default_rng(41)
    for causal, (nq, H, dn, dr, L) in [(True, (3, 4, 6, 4, 23)), (False, (2, 3, 5, 6, 17)),
                                       (True, (1, 2, 3, 2, 9))]:
        qn, qp = rng.standard_normal((nq, H, dn)), rng.standard_normal((nq, H, dr))
        kn, kp = rng.standard_normal((L, dn)), rng.standard_normal((L, dr))
        theta = rng.uniform(0.05, 1.2, size=dr // 2)
        q_pos = np.arange(L - nq, L)
        scale = 0.61
        got = O.kv_shared_reference(qn, qp, kn, kp, theta, q_pos, scale, causal=causal)
        h = dr // 2
        perm = np.empty(dr, dtype=np.int64)              # half-split index -> interleaved slot
        perm[0::2], perm[1::2] = np.arange(h), np.arange(h) + h
        q = np.concatenate([qn, _complex_rotate(qp[..., perm], theta, q_pos[:, None])], -1)
        kv = np.concatenate([kn, _complex_rotate(kp[..., perm], theta, np.arange(L))], -1)
        qt = torch.from_numpy(q).permute(1, 0, 2)[None]                    # [1, H, q, Dh]
        kt = torch.from_numpy(kv)[None, None].expand(1, H, L, dn + dr)
        mask = torch.from_numpy(np.arange(L)[None, :] <= q_pos[:, None]) if causal else None
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mask,
                                                             scale=scale)[0].permute(1, 0, 2).numpy()
        o = o.copy()
        o[..., dn:] = _complex_rotate(o[..., dn:], theta, -q_pos[:, None])
        inv = np.argsort(perm)
        o[..., dn:] = o[..., dn:][..., inv]
        _close(got["o"], o, 1e-12, "kv-shared o vs sdpa")
        s = torch.einsum("hid,ld->ihl", qt[0], torch.from_numpy(kv)) * scale
        if causal:
            s = s.masked_fill(~mask[:, None, :], float("-inf"))
        _close(got["lse"], torch.logsumexp(s, dim=-1).numpy(), 1e-12, "kv-shared lse")


def pin_kv_shared_single_token(O):
    """One cached token at position 0 and a query at position 0: the output is that token's
    vector itself (the rotation at position 0 is the identity), lse its scaled score."""
    rng = np.random.default_rng(43)
    qn, qp = rng.standard_normal((1, 3, 5)), rng.standard_normal((1, 3, 4))
    kn, kp = rng.standard_normal((1, 5)), rng.standard_normal((1, 4))
    got = O.kv_shared_reference(qn, qp, kn, kp, np.array([0.3, 0.9]), np.array([0]), 0.5)
    want = np.concatenate([kn, kp], -1)[None].repeat(3, axis=1)
    _close(got["o"], want, 1e-14, "single token o")
    s = 0.5 * (np.einsum("ihd,d->ih", qn, kn[0]) + np.einsum("ihd,d->ih", qp, kp[0]))
    _close(got["lse"], s, 1e-14, "single token lse")


def pin_absorbed_baseline(O):
    """The absorbed-order CPU baseline equals the unabsorbed definition (associativity of
    einsums (1)-(3) against (4)-(5)) and the scalar brute force."""
    for seed, kw in [(51, dict(nq=2, H=6, G=3, r=5, dn=4, dr=4, dv=3, L=11)),
                     (52, dict(nq=1, H=4, G=1, r=8, dn=3, dr=2, dv=6, L=7, bias=False))]:
        P = _problem(seed, **kw)
        got = O.mla_decode_absorbed(**P)
        ref = _brute_force(**P)
        for k in ("o", "o_latent", "lse"):
            _close(got[k], ref[k], 1e-11, f"absorbed baseline {k}")


def pin_down_kv_bruteforce(O):
    """The down-projection against literal loops over tokens, outputs and the hidden dim,
    and the split of its output into the latent and each group's rotary key."""
    rng = np.random.default_rng(61)
    B, n, hid, r, G, dr = 2, 3, 7, 4, 2, 2
    x = rng.standard_normal((B, n, hid))
    w = rng.standard_normal((r + G * dr, hid))
    c_kv, k_r = O.down_kv_reference(x, w, r, G, dr)
    for b in range(B):
        for t in range(n):
            for d in range(r + G * dr):
                acc = 0.0
                for k in range(hid):
                    acc += w[d][k] * x[b][t][k]
                got = c_kv[b, t, d] if d < r else k_r[b, t, (d - r) // dr, (d - r) % dr]
                assert abs(got - acc) <= 1e-12 * max(1.0, abs(acc)), (b, t, d)


def pin_o_proj_original_order(O):
    """Einsum (6) after (4)-(5) equals einsum (3) of the original order, computed from the
    up-projected values and the attention weights with literal loops: u[i, D] = sum over h, d
    of W_o[h, d, D] * sum_l p[i, h, l] * V_h[l, d]."""
    P = _problem(71, nq=2, H=3, G=1, r=4, dn=2, dr=2, dv=3, L=5, bias=False)
    rng = np.random.default_rng(72)
    hid = 4
    w_o = rng.standard_normal((3, 3, hid))
    b_o = rng.standard_normal(hid)
    got = O.mla_decode_reference(want_p=True, **P)
    u = O.o_proj_reference(O.out_up_reference(got["o_latent"], P["w_uv"]), w_o, b_o)
    p = got["p"]
    for i in range(2):
        for D in range(hid):
            acc = b_o[D]
            for h in range(3):
                for d in range(3):
                    v = 0.0
                    for l in range(5):
                        vl = sum(P["w_uv"][h][d][c] * P["c_kv"][l][c] for c in range(4))
                        v += p[i][h][l] * vl
                    acc += w_o[h][d][D] * v
            assert abs(u[i, D] - acc) <= 1e-11 * max(1.0, abs(acc)), (i, D)


ALL_PINS = [pin_absorb_single_token, pin_out_up_associativity, pin_bruteforce, pin_associativity, pin_sdpa_identity_weights, pin_zero_query_uniform,
            pin_single_token, pin_rows_sum_to_one, pin_causal_prefix, pin_rope_complex,
            pin_rope_norm_and_relative, pin_bf16_rounding, pin_rotate_fp32, pin_append_slots,
            pin_kv_shared_sdpa, pin_kv_shared_single_token, pin_absorbed_baseline,
            pin_down_kv_bruteforce, pin_o_proj_original_order]
