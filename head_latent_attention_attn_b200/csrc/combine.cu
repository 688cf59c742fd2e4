// combine.cu - the merge of sequences cut between CTAs by mla_decode_attn's schedule: each
// piece left its normalised partial o (bf16) and lse (fp32); the row's
//   lse = log sum_i e^{lse_i},   o = sum_i e^{lse_i - lse} o_i
// (the log-sum-exp identity) is written to o_latent and lse.
#include <math.h>

#include <algorithm>

#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

// Bring `bytes` (a multiple of 16) at the 16-byte-aligned global address `src` into L2.
MLA_DEVICE void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Before its grid-dependency wait, block i of the merge brings slice i of p.l2_prefetch into
// L2 (the blocks start as the decode's CTAs leave, so this overlaps the decode's last CTAs).
MLA_DEVICE void prefetch_next_weights(const CombineParams& p) {
  if (p.l2_prefetch == nullptr || threadIdx.x != 0) return;
  const int64_t slice = ((p.l2_prefetch_bytes + gridDim.x - 1) / gridDim.x + 15) & ~int64_t(15);
  const int64_t off = int64_t(blockIdx.x) * slice;
  const int64_t n = min(slice, p.l2_prefetch_bytes - off) & ~int64_t(15);
  for (int64_t o = 0; o < n; o += 65536)
    bulk_prefetch_l2(static_cast<const uint8_t*>(p.l2_prefetch) + off + o,
                     uint32_t(min(int64_t(65536), n - o)));
}

// ---- merge of cut units: lse = log sum_i e^{lse_i}, o = sum_i e^{lse_i - lse} o_i ------
// One block per (unit, query row): warp 0 reduces the pieces' lse, then the 4 warps split
// the pieces and every lane accumulates up to 16 latents (8 x lane + 256 k + 0..7: one
// 16-byte load of a piece's bf16 row per k; two pieces' loads in flight per step); shared
// memory adds the warps.
__global__ void __launch_bounds__(128) mla_combine_kernel(const CombineParams p) {
  __shared__ float part[4][512];
  __shared__ float lse_s;
  prefetch_next_weights(p);
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = int(blockIdx.x / unsigned(p.ncol));
  const int n = int(blockIdx.x % unsigned(p.ncol));
  const int G = p.col_groups;
  const int b = u / G, cg = u - b * G;
  const int f = cg * p.ncol + n;
  if (f >= p.qH) return;
  int L = p.seq_lens[b];
  const bool ok = L >= p.q_len && L <= p.max_seq_len && int64_t(L) <= int64_t(p.max_pages) * kDecodeTok;
  if (!ok) L = 0;
  const int tiles = L > 0 ? (L + kDecodeTok - 1) / kDecodeTok : 1;
  const int per = *p.range_len;
  const int s = p.unit_start[u];
  const int i0 = s / per, i1 = (s + tiles - 1) / per;
  if (i0 == i1) return;   // held whole by one CTA: already written
  if (warp == 0) {
    float mx = -INFINITY;
    for (int i = i0 + lane; i <= i1; i += 32)
      mx = fmaxf(mx, p.part_lse[int64_t(piece_slot(i, s, per, G, cg)) * p.ncol + n]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.0f;
    for (int i = i0 + lane; i <= i1; i += 32) {
      const float li = p.part_lse[int64_t(piece_slot(i, s, per, G, cg)) * p.ncol + n];
      den += li == -INFINITY ? 0.0f : expf(li - mx);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) lse_s = mx == -INFINITY ? -INFINITY : mx + logf(den);
  }
  __syncthreads();
  const float lse = lse_s;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
  // latents 8 * lane + 256 * k + e of a piece's row: 16-byte aligned (r % 8 == 0)
  auto add_piece = [&](int i) {
    const int64_t sl = piece_slot(i, s, per, G, cg);
    const float li = p.part_lse[sl * p.ncol + n];
    const uint16_t* row = p.part_o + (sl * p.ncol + n) * p.r;
    uint4 v[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int lat = 8 * lane + 256 * k;
      v[k] = (lat < p.r && li != -INFINITY) ? *reinterpret_cast<const uint4*>(row + lat)
                                            : make_uint4(0u, 0u, 0u, 0u);
    }
    const float wgt = li == -INFINITY ? 0.0f : expf(li - lse);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[8 * k + 2 * e] += wgt * __uint_as_float(w[e] << 16);
        acc[8 * k + 2 * e + 1] += wgt * __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  };
  int i = i0 + warp;
  for (; i + 4 <= i1; i += 8) {
    add_piece(i);
    add_piece(i + 4);
  }
  if (i <= i1) add_piece(i);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int lat = 8 * lane + 256 * k;
    if (lat < p.r) {
#pragma unroll
      for (int e = 0; e < 8; ++e) part[warp][lat + e] = acc[8 * k + e];
    }
  }
  __syncthreads();
  uint16_t* out = p.o_latent + (int64_t(b) * p.qH + f) * p.r;
  for (int lat = threadIdx.x; lat < p.r; lat += 128)
    out[lat] = f32_to_bf16_rne(part[0][lat] + part[1][lat] + part[2][lat] + part[3][lat]);
  if (threadIdx.x == 0) p.lse[int64_t(b) * p.qH + f] = lse;
}

// The same merge with one warp per (unit, query row), for units cut into a few pieces: a
// grid of 256-thread blocks (8 warps) sized to fill the GPU once, each warp looping over
// rows. Lane i reads piece i's lse; lanes own latents 4 * lane + 128 k, so every load of a
// piece's bf16 row is one 256-byte coalesced segment per warp. For up to kFewPieces pieces
// the rows of all pieces are loaded together with their lse (one round trip to L2 after
// the schedule's), and the weights come from shuffles; more pieces take a loop.
constexpr int kFewPieces = 4;

__global__ void __launch_bounds__(256) mla_combine_rows_kernel(const CombineParams p) {
  prefetch_next_weights(p);
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t nrows = int64_t(p.units) * p.ncol;
  const int64_t nwarps = int64_t(gridDim.x) * 8;
  const int G = p.col_groups;
  const int per = *p.range_len;
  for (int64_t gw = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5); gw < nrows; gw += nwarps) {
    const int u = int(gw / p.ncol);
    const int n = int(gw - int64_t(u) * p.ncol);
    const int b = u / G, cg = u - b * G;
    const int f = cg * p.ncol + n;
    if (f >= p.qH) continue;
    int L = p.seq_lens[b];
    const bool okL = L >= p.q_len && L <= p.max_seq_len &&
                     int64_t(L) <= int64_t(p.max_pages) * kDecodeTok;
    if (!okL) L = 0;
    const int tiles = L > 0 ? (L + kDecodeTok - 1) / kDecodeTok : 1;
    const int s = p.unit_start[u];
    const int i0 = s / per, i1 = (s + tiles - 1) / per;
    if (i0 == i1) continue;   // held whole by one range: already written
    const int np = i1 - i0 + 1;
    float acc[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[k][e] = 0.0f;
    float lse;
    if (np <= kFewPieces) {
      // every load at once: lse of piece `lane`, and each piece's row chunks
      const float my_l = lane < np
                             ? p.part_lse[int64_t(piece_slot(i0 + lane, s, per, G, cg)) * p.ncol + n]
                             : -INFINITY;
      uint2 v[kFewPieces][4];
#pragma unroll
      for (int i = 0; i < kFewPieces; ++i) {
        const uint16_t* row =
            p.part_o + (int64_t(piece_slot(i0 + min(i, np - 1), s, per, G, cg)) * p.ncol + n) * p.r;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int lat = 4 * lane + 128 * k;
          v[i][k] = (i < np && lat < p.r) ? *reinterpret_cast<const uint2*>(row + lat)
                                          : make_uint2(0u, 0u);
        }
      }
      float mx = my_l;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float den = my_l == -INFINITY ? 0.0f : expf(my_l - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      lse = mx == -INFINITY ? -INFINITY : mx + logf(den);
#pragma unroll
      for (int i = 0; i < kFewPieces; ++i) {
        const float li = __shfl_sync(0xffffffffu, my_l, i);
        const float wgt = (i < np && li != -INFINITY) ? expf(li - lse) : 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[k][0] += wgt * __uint_as_float(v[i][k].x << 16);
          acc[k][1] += wgt * __uint_as_float(v[i][k].x & 0xFFFF0000u);
          acc[k][2] += wgt * __uint_as_float(v[i][k].y << 16);
          acc[k][3] += wgt * __uint_as_float(v[i][k].y & 0xFFFF0000u);
        }
      }
    } else {
      float mx = -INFINITY;
      for (int i = i0 + lane; i <= i1; i += 32)
        mx = fmaxf(mx, p.part_lse[int64_t(piece_slot(i, s, per, G, cg)) * p.ncol + n]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float den = 0.0f;
      for (int i = i0 + lane; i <= i1; i += 32) {
        const float li = p.part_lse[int64_t(piece_slot(i, s, per, G, cg)) * p.ncol + n];
        den += li == -INFINITY ? 0.0f : expf(li - mx);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      lse = mx == -INFINITY ? -INFINITY : mx + logf(den);
      for (int i = i0; i <= i1; ++i) {
        const int64_t sl = piece_slot(i, s, per, G, cg);
        const float li = p.part_lse[sl * p.ncol + n];
        if (li == -INFINITY) continue;
        const float wgt = expf(li - lse);
        const uint16_t* row = p.part_o + (sl * p.ncol + n) * p.r;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int lat = 4 * lane + 128 * k;
          if (lat < p.r) {
            const uint2 x = *reinterpret_cast<const uint2*>(row + lat);   // r % 4 == 0
            acc[k][0] += wgt * __uint_as_float(x.x << 16);
            acc[k][1] += wgt * __uint_as_float(x.x & 0xFFFF0000u);
            acc[k][2] += wgt * __uint_as_float(x.y << 16);
            acc[k][3] += wgt * __uint_as_float(x.y & 0xFFFF0000u);
          }
        }
      }
    }
    uint16_t* out = p.o_latent + (int64_t(b) * p.qH + f) * p.r;
    const bool vec = (reinterpret_cast<uintptr_t>(out) & 7u) == 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int lat = 4 * lane + 128 * k;
      if (lat >= p.r) continue;
      if (vec) {
        *reinterpret_cast<uint2*>(out + lat) = make_uint2(cvt_bf16x2(acc[k][0], acc[k][1]),
                                                          cvt_bf16x2(acc[k][2], acc[k][3]));
      } else {
        out[lat] = f32_to_bf16_rne(acc[k][0]);
        out[lat + 1] = f32_to_bf16_rne(acc[k][1]);
        out[lat + 2] = f32_to_bf16_rne(acc[k][2]);
        out[lat + 3] = f32_to_bf16_rne(acc[k][3]);
      }
    }
    if (lane == 0) p.lse[int64_t(b) * p.qH + f] = lse;
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const int64_t rows = int64_t(p.units) * p.ncol;
  if (rows <= 0 || rows > 0x7fffffffLL || p.r > 512 || p.r % 4 != 0) return cudaErrorInvalidValue;
  if (int64_t(p.vgrid) <= 4 * int64_t(p.units)) {
    // a few pieces per unit: one warp per row
    // 8 rows per block at a time; at most 4 blocks per SM (all resident at once)
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, int64_t(std::max(p.sms, 1)) * 4);
    return launch_pdl(mla_combine_rows_kernel, dim3(unsigned(blocks)), dim3(256), 0, stream, 1,
                      p);
  }
  // many pieces per unit: the four warps of a block split one row's pieces
  return launch_pdl(mla_combine_kernel, dim3(unsigned(rows)), dim3(128), 0, stream, 1, p);
}

}  // namespace mla
