// append.cuh - one new token's cache row, written by one warp: the latent row moves as
// 16-byte vectors, the rotary pairs are rotated in fp32 (separately rounded multiply /
// subtract / add) and rounded to bf16 with ties to even. Used by cache_append_kernel and,
// folded into the query absorption, by the one-call decode step.
#pragma once

#include "kernels.h"
#include "ptx.cuh"

namespace mla {

// Token gw = b * n_new + t of the batch (0 <= gw < batch * n_new); all 32 lanes call it.
MLA_DEVICE void append_token(const AppendParams& p, int64_t gw, int lane) {
  const int b = int(gw / p.n_new);
  const int t = int(gw - int64_t(b) * p.n_new);
  const int64_t pos = int64_t(p.start_pos[b]) + t;
  const int64_t lp = pos >= 0 ? pos / p.page_size : -1;
  if (pos < 0 || lp >= p.max_pages) {
    if (lane == 0 && p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
    return;
  }
  const int32_t page = p.block_table[int64_t(b) * p.max_pages + lp];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0 && p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
    return;
  }
  const int D = p.r + p.groups * p.rope_dim;
  uint16_t* dst = p.cache + (int64_t(page) * p.page_size + pos % p.page_size) * D;

  // latent: exact copy, 8 bf16 per 16-byte vector (r % 8 == 0, rows 16-byte aligned)
  const uint4* src4 = reinterpret_cast<const uint4*>(p.c_kv + gw * p.r);
  uint4* dst4 = reinterpret_cast<uint4*>(dst);
  for (int i = lane; i < p.r / 8; i += 32) dst4[i] = src4[i];

  // rotary key of every group
  const int half = p.rope_dim / 2;
  const int npairs = p.groups * half;
  const uint16_t* kr = p.k_r + gw * int64_t(p.groups) * p.rope_dim;
  const float* cs = p.rope_cos + gw * npairs;
  const float* sn = p.rope_sin + gw * npairs;
  for (int idx = lane; idx < npairs; idx += 32) {
    const int g = idx / half;
    const int j = idx - g * half;
    const float x0 = bf16_bits_to_f32(kr[g * p.rope_dim + j]);
    const float x1 = bf16_bits_to_f32(kr[g * p.rope_dim + j + half]);
    const float c = cs[idx];
    const float s = sn[idx];
    const float y0 = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
    const float y1 = __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
    dst[p.r + g * p.rope_dim + j] = f32_to_bf16_rne(y0);
    dst[p.r + g * p.rope_dim + j + half] = f32_to_bf16_rne(y1);
  }
}

}  // namespace mla
