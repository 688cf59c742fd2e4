"""GPU test harness: the device-resident problem plus its comparisons with the oracle.

``GpuProblem`` is ``mla_inputs.device.DeviceProblem`` (inputs on the GPU, the decode step
through the library's C ABI) with methods that run the fp64 CPU oracle on the same seeded
inputs; ``check_sequence`` applies the parity tolerances.
"""
from __future__ import annotations

import numpy as np

from mla_inputs.device import DeviceProblem, dims_of  # noqa: F401


class GpuProblem(DeviceProblem):
    def oracle(self, b: int):
        import oracle.mla_oracle as O  # test infrastructure only
        wl = self.wl
        c_kv, k_r = wl.context(b)
        return O.mla_decode_reference(wl.q_nope[b], wl.q_pe[b], c_kv, k_r, wl.w_uk, wl.w_uv,
                                      wl.bias, wl.theta, wl.query_positions()[b],
                                      self.cfg.softmax_scale, causal=self.cfg.causal)

    def oracle_heads(self, b: int, heads) -> dict:
        """The oracle for sequence b restricted to some heads: {h: {"o", "o_latent", "lse"}}
        with arrays over the q query rows. Heads are independent in the oracle, so the
        inputs are sliced per key group (the heads of one group see one k_r slice)."""
        import oracle.mla_oracle as O  # test infrastructure only
        wl, cfg = self.wl, self.cfg
        c_kv, k_r = wl.context(b)
        g_of = O.group_of_head(cfg.num_heads, cfg.num_kv_groups)
        out = {}
        for g in sorted({int(g_of[h]) for h in heads}):
            hs = [int(h) for h in heads if int(g_of[h]) == g]
            bias = None if wl.bias is None else wl.bias[hs]
            ref = O.mla_decode_reference(wl.q_nope[b][:, hs], wl.q_pe[b][:, hs], c_kv,
                                         k_r[:, g:g + 1], wl.w_uk[hs], wl.w_uv[hs], bias,
                                         wl.theta[g:g + 1], wl.query_positions()[b],
                                         cfg.softmax_scale, causal=cfg.causal)
            for j, h in enumerate(hs):
                out[h] = {k: ref[k][:, j] for k in ("o", "o_latent", "lse")}
        return out


def max_rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max|got - ref| / max|ref| (the tolerance measure of the parity tests)."""
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


O_TOL = 2e-2      # max|o - o_ref| <= 2e-2 * max|o_ref|
LSE_TOL = 1e-3    # |lse - lse_ref| <= 1e-3 (absolute)


def check_sequence(prob: GpuProblem, b: int, what: str = "") -> dict:
    ref = prob.oracle(b)
    o = prob.o[b].float().cpu().numpy()
    ol = prob.o_latent[b].float().cpu().numpy()
    lse = prob.lse[b].float().cpu().numpy()
    res = {
        "o": max_rel_err(o, ref["o"]),
        "o_latent": max_rel_err(ol, ref["o_latent"]),
        "lse": float(np.max(np.abs(lse - ref["lse"]))),
    }
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ol)) and np.all(np.isfinite(lse)), \
        f"{what} seq {b}: non-finite output"
    assert res["o"] <= O_TOL, f"{what} seq {b}: o rel err {res['o']:.3e}"
    assert res["o_latent"] <= O_TOL, f"{what} seq {b}: o_latent rel err {res['o_latent']:.3e}"
    assert res["lse"] <= LSE_TOL, f"{what} seq {b}: lse err {res['lse']:.3e}"
    return res
