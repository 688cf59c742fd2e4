"""CPU fp64 oracle for MLA decode. Test infrastructure: never imported by the product."""
from .mla_oracle import (  # noqa: F401
    absorb_reference, as_f64, out_up_reference, bf16_bits_to_f32, cache_append_emulate, f32_to_bf16_bits, group_of_head,
    mla_decode_reference, rope_rotate, rotate_fp32, kv_shared_reference, mla_decode_absorbed, down_kv_reference, o_proj_reference,
)
