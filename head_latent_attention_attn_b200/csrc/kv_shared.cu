// kv_shared.cu - the two elementwise steps of the single-latent K = V form (nanowhale-100m
// page, cnnetsun.cn: one head_dim vector per token is both key and value, with RoPE on its
// last d_r dims, and the output's rotary dims are rotated back after attention).
//
// In that form the cache row [nope (r) | rotated rope (d_r)] is the whole key AND the whole
// value, so the attention itself is mla_decode_attn over rows of width D = r + d_r with no
// separate rotary slot. Around it:
//   query:  q_ext[row, :r] = q[row, :r];  q_ext[row, r:] = R(pos) q[row, r:]
//   output: o[row, :r]     = o_[row, :r]; o[row, r:]     = R(-pos) o_[row, r:]
// where R(pos) rotates the pairs (x_j, x_{j+d_r/2}) by theta_j * pos (cos/sin tables from
// the caller, fp32), computed in fp32 with separately rounded products and sums and
// rounded to bf16 with ties to even. One warp per (b, i, h) row: the first r elements move
// as 16-byte vectors, the rotary pairs one pair per lane.
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

__global__ void __launch_bounds__(256) kv_shared_rotate_kernel(KvSharedParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const int D = p.r + p.rope_dim;
  const int64_t bq = row / p.heads;                 // (b, i): the row's query token
  const uint16_t* src = p.in + row * D;
  uint16_t* dst = p.out + row * D;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int k = lane; k < p.r / 8; k += 32) d4[k] = s4[k];
  const int half = p.rope_dim / 2;
  const float* cs = p.rope_cos + bq * half;
  const float* sn = p.rope_sin + bq * half;
  for (int j = lane; j < half; j += 32) {
    const float x0 = bf16_bits_to_f32(src[p.r + j]);
    const float x1 = bf16_bits_to_f32(src[p.r + j + half]);
    const float c = cs[j];
    const float s = p.inverse ? -sn[j] : sn[j];     // R(-pos): the same angle, negated sine
    const float y0 = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
    const float y1 = __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
    dst[p.r + j] = f32_to_bf16_rne(y0);
    dst[p.r + j + half] = f32_to_bf16_rne(y1);
  }
}

cudaError_t launch_kv_shared_rotate(const KvSharedParams& p, cudaStream_t stream) {
  if (p.rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (p.rows * 32 + threads - 1) / threads;
  return launch_pdl(kv_shared_rotate_kernel, dim3(unsigned(blocks)), dim3(threads), 0, stream, 1,
                    p);
}

}  // namespace mla
