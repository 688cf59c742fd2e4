"""Plant plausible mistakes in copies of the oracle and check that a pin catches each.

A mutation is a textual edit of the oracle's source (a dropped term, a wrong sign,
index or operand); the edited source is executed as a fresh module and the pins of
tests/oracle_pins.py run against it. Every mutation must fail at least one pin.
"""
import inspect
import types

import pytest

import oracle.mla_oracle as O
from tests.oracle_pins import ALL_PINS

MUTATIONS = {
    "dropped_softmax_scale": ("softmax_scale * (Q @ K.T)", "(Q @ K.T)"),
    "rope_sign": ("x0 * c - x1 * s", "x0 * c + x1 * s"),
    "rope_interleaved_pairs": ("x0, x1 = x[..., :h], x[..., h:]", "x0, x1 = x[..., 0::2], x[..., 1::2]"),
    "causal_off_by_one": ("tok_pos[None, :] <= q_pos[:, None]", "tok_pos[None, :] < q_pos[:, None]"),
    "wrong_key_weight": ("c_kv[l0:l1] @ w_uk[h].T", "c_kv[l0:l1] @ w_uv[h].T"),
    "bias_sign": ("V = V + bias[h]", "V = V - bias[h]"),
    "dropped_rope_term": ("K = np.concatenate([K_nope, k_rot[l0:l1, g_of[h], :]], axis=-1)",
                          "K = np.concatenate([K_nope, 0.0 * k_rot[l0:l1, g_of[h], :]], axis=-1)"),
    "group_always_zero": ("k_rot[l0:l1, g_of[h], :]", "k_rot[l0:l1, 0, :]"),
    "group_mapping_modulo": ("np.arange(num_heads) // (num_heads // num_groups)",
                             "np.arange(num_heads) % num_groups"),
    "query_position_shift": ("theta[g_of[h]], q_pos)", "theta[g_of[h]], q_pos + 1)"),
    "key_position_shift": ("theta[g], tok_pos)", "theta[g], tok_pos + 1)"),
    "lse_log2": ("m[:, 0] + np.log(", "m[:, 0] + np.log2("),
    "latent_uses_values": ("acc_c += p[:, l0:l1] @ c_kv[l0:l1]", "acc_c += p[:, l0:l1] @ (2 * c_kv[l0:l1])"),
    "round_half_up": ("((u + 0x7FFF + lsb) >> 16)", "((u + 0x8000) >> 16)"),
    "truncate_not_round": ("((u + 0x7FFF + lsb) >> 16)", "((u) >> 16)"),
    "fp32_rotation_sign": ("y1 = np.add(", "y1 = np.subtract("),
    "append_row_shift": ("rows = pos % page_size", "rows = (pos + 1) % page_size"),
    "append_page_index": ("pages = block_table[b, pos // page_size]", "pages = block_table[b, pos // page_size * 0]"),
    "absorb_wrong_contraction": ('np.einsum("hdc,ihd->ihc", w_uk, q_nope)', 'np.einsum("hdc,ihd->ihc", w_uk, q_nope[:, ::-1])'),
    "out_up_bias_dropped": ("        o = o + as_f64(bias)", "        o = o + 0.0"),
    "append_groups_swapped": ("out[pages, rows, r:] = f32_to_bf16_bits(y).reshape(n, G * dr)",
                              "out[pages, rows, r:] = f32_to_bf16_bits(y[:, ::-1]).reshape(n, G * dr)"),
    "kv_shared_no_inverse_rotation": ("o[..., dn:] = rope_rotate(o[..., dn:], theta, -q_pos[:, None])",
                                      "o[..., dn:] = o[..., dn:]"),
    "kv_shared_inverse_sign": ("o[..., dn:] = rope_rotate(o[..., dn:], theta, -q_pos[:, None])",
                               "o[..., dn:] = rope_rotate(o[..., dn:], theta, q_pos[:, None])"),
    "kv_shared_value_unrotated": ('o = np.einsum("ihl,ld->ihd", p, kv)',
                                  'o = np.einsum("ihl,ld->ihd", p, np.concatenate([kv_nope, kv_pe], -1))'),
    "kv_shared_query_unrotated": ("Q = np.concatenate([q_nope, q_rot], axis=-1)",
                                  "Q = np.concatenate([q_nope, q_pe], axis=-1)"),
    "absorbed_dropped_rope_term": ('np.einsum("ihe,le->ihl", q_rot[:, hs], k_rot))',
                                   '0.0 * np.einsum("ihe,le->ihl", q_rot[:, hs], k_rot))'),
    "down_kv_transposed_weight": ('np.einsum("...k,dk->...d", as_f64(hidden), as_f64(w_dkv))',
                                  'np.einsum("...k,dk->...d", as_f64(hidden), as_f64(w_dkv)[::-1])'),
    "down_kv_split_off_by_one": ("k_r = out[..., kv_lora_rank:]", "k_r = out[..., kv_lora_rank - 1:-1]"),
    "o_proj_transposed_head_dims": ('np.einsum("...hd,hdk->...k", as_f64(o), as_f64(w_o))',
                                    'np.einsum("...hd,hdk->...k", as_f64(o)[..., ::-1], as_f64(w_o))'),
}


def _mutant(old: str, new: str) -> types.ModuleType:
    src = inspect.getsource(O)
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    old, new = MUTATIONS[name]
    mod = _mutant(old, new)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts as caught
            caught.append(f"{pin.__name__}: {type(e).__name__}")
    assert caught, f"mutation {name} passed every pin"


def test_unmutated_copy_passes():
    mod = _mutant("import numpy as np", "import numpy as np")
    for pin in ALL_PINS:
        pin(mod)
