// kernels.h - parameter blocks and launchers of the sm_100a kernels behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace mla {

// Launch `kernel` with programmatic dependent launch (it may start while the previous kernel
// on `stream` runs; see grid_dep_wait in ptx.cuh) and, when cluster_x > 1, clusters of
// cluster_x CTAs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = unsigned(cluster_x);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = unsigned(n);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---- mla_cache_append -------------------------------------------------------------------
struct AppendParams {
  const uint16_t* c_kv;      // [B, n_new, r]
  const uint16_t* k_r;       // [B, n_new, G, d_r]
  const float* rope_cos;     // [B, n_new, G, d_r/2]
  const float* rope_sin;
  const int32_t* block_table;
  const int32_t* start_pos;
  uint16_t* cache;           // [num_pages, ps, D]
  int32_t* dev_error;
  int64_t num_pages;
  int32_t max_pages, batch, n_new, r, groups, rope_dim, page_size;
};
cudaError_t launch_cache_append(const AppendParams& p, cudaStream_t stream);

// ---- the single-latent K = V form: rotary slice of the query / inverse rotation of o ---
struct KvSharedParams {
  const uint16_t* in;        // [rows, r + d_r] bf16
  uint16_t* out;             // [rows, r + d_r] bf16 (may equal `in`)
  const float* rope_cos;     // [rows / heads, d_r / 2]
  const float* rope_sin;
  int64_t rows;              // B * q * H
  int32_t heads, r, rope_dim;
  int32_t inverse;           // 0: rotate by +pos (query), 1: by -pos (output)
};
cudaError_t launch_kv_shared_rotate(const KvSharedParams& p, cudaStream_t stream);

// ---- per-head weight GEMM (mla_absorb_q, mla_out_up) --------------------------------------
// For every head h and activation row n: out[n, h, m] = sum_k W_h[m, k] * x[n, h, k] (+ bias).
// The weight tile is the UMMA A operand (M = output features), the activation rows are B.
struct WGemmParams {
  CUtensorMap tm_w;          // 3D weight map, box 128 x 64 (see launcher)
  CUtensorMap tm_x;          // 3D activations {K, H, rows}, box {64, 1, NR}
  uint16_t* out;             // element (n, h, m) at n*out_row_stride + h*out_head_stride + m
  CUtensorMap tm_out;        // 3D {M, H, rows} over out, box {128, 1, NR} (clipped past M)
  int64_t out_row_stride, out_head_stride;
  const uint16_t* bias;      // [H, M] or null
  int32_t* dev_error;
  int32_t M, K, rows, heads;
  int32_t a_mn;              // 1: weight stored [K][M] (W_UK), 0: stored [M][K] (W_UV)
  int32_t tma_out;           // 1: tm_out stores the output tiles (else element copies)
  // rotary part of q_ext (mla_absorb_q only; q_pe == nullptr otherwise)
  const uint16_t* q_pe;      // [rows, H, d_r]
  const float* rope_cos;     // [rows, G, d_r/2]
  const float* rope_sin;
  int32_t groups, rope_dim;
  int32_t rope_vec;          // 1: q_pe 8-byte, cos/sin 16-byte aligned and d_r/2 % 4 == 0
  // cache append folded into the absorption (the one-call decode step; batch == 0 when
  // unused): the epilogue warps write the new tokens' cache rows before their first item
  AppendParams app;
};
// max_ctas: the persistent grid's size limit (one CTA per SM).
cudaError_t launch_wgemm(const WGemmParams& p, int nr, int max_ctas, cudaStream_t stream);

// ---- mla_down_kv_append: split-K GEMM on clusters, cache rows in the epilogue (down_kv.cu)
struct DkvParams {
  CUtensorMap tm_w;          // 2D {hidden, D} over w_dkv, box {64, 128}
  CUtensorMap tm_x;          // 2D {hidden, rows} over the hidden states, box {64, NR}
  uint16_t* cache;           // [num_pages, page_size, D]
  const int32_t* block_table;   // [B, max_pages]
  const int32_t* start_pos;     // [B]
  const float* rope_cos;     // [rows, G, d_r/2]
  const float* rope_sin;
  uint16_t* kv_out;          // [rows, D] or null
  int32_t* dev_error;
  int64_t num_pages;
  int32_t max_pages, n_new, page_size, r, groups, rope_dim, rows, K;
  int32_t lat_tiles;         // ceil(r / 128) latent feature tiles (+ one rotary tile)
  int32_t n_nt;              // row tiles of NR tokens
  int32_t splits;            // CTAs per cluster splitting K (the cluster size)
};
cudaError_t launch_down_kv(const DkvParams& p, int nr, cudaStream_t stream);

// ---- mla_out_proj: einsum (5) then einsum (6) in one cooperative kernel (oproj.cu) -------
struct OProjParams {
  CUtensorMap tm_wuv;        // 3D {r, d_v, H} (head stride), box {64, 128, 1}
  CUtensorMap tm_ol;         // 3D {r, H, rows}, box {64, 1, NR}: o_latent
  CUtensorMap tm_wo;         // 2D {H*d_v, hidden}, box {64, 128}: W_o as [hidden][H*d_v]
  CUtensorMap tm_o;          // 2D {H*d_v, rows}, box {64, NR}: stage A's output o
  uint16_t* o;               // [rows, H, d_v] bf16 (stage A output, stage B input)
  uint16_t* u;               // [rows, hidden] bf16
  const uint16_t* bias_v;    // [H, d_v] or null
  const uint16_t* bias_o;    // [hidden] or null
  float* part;               // [splits, rows, hidden] fp32 partials of stage B
  int32_t* head_done;        // [H] stage-A items done per head (cleared by the kernel)
  int32_t* tile_done;        // [tiles] stage-B splits done per output tile (cleared)
  int32_t* cta_done;         // [1] CTAs finished (cleared)
  int32_t* dev_error;
  int32_t H, r, dv, hidden, rows, splits;
};
size_t oproj_smem_bytes(int nr);
cudaError_t launch_oproj(const OProjParams& p, int nr, int grid, cudaStream_t stream);

// ---- mla_decode_attn -----------------------------------------------------------------------
constexpr int kDecodeTok = 64;        // tokens per tile = one cache page
constexpr int kDecodeMaxBlk = 10;     // D <= 640 -> at most 10 64-column blocks
constexpr int kDecodeMaxSlots = 8;

struct DecodeParams {
  CUtensorMap tm_cache;      // 2D {D, num_pages*64}, box {64, 64}, 128B swizzle
  CUtensorMap tm_q;          // 3D {D, q*H, B}, box {64, NCOL, 1}, 128B swizzle
  const int32_t* block_table;
  const int32_t* seq_lens;
  uint16_t* o_latent;        // [B, q, H, r]
  float* lse;                // [B, q, H]
  uint16_t* part_o;          // [grid, 2, NCOL, r]  partial outputs of cut units (bf16)
  float* part_lse;           // [grid, 2, NCOL]
  int32_t* unit_start;       // [units] first tile of each unit in its row block (for the merge)
  int32_t* range_len;        // [1] tiles per CTA range (for the merge)
  int32_t* dev_error;
  int64_t num_pages;
  int32_t max_pages, batch, q_len, num_heads, qH, r, D, nblk, nch, col_groups, units,
      max_seq_len, causal, nslot, slot_blocks, tmem_cols, npt;
  float scale_log2;          // softmax_scale * log2(e)
  // used by the latent-split cluster kernel only
  CUtensorMap tm_rope;       // 2D {D, num_pages*64}, box {rope_half, 64}
  const uint16_t* q_ext;     // [B, q*H, D]
  int32_t rope_half;         // rotary columns per CTA of the pair (G*d_r/2)
};
size_t decode_smem_bytes(int ncol, int nblk, int slot_blocks, int nslot, int npt);
cudaError_t launch_decode(const DecodeParams& p, int ncol, dim3 grid, size_t smem,
                          cudaStream_t stream);

// Blocks of up to 128 query rows: a cluster of two CTAs splits the latent (decode_pair.cu).
constexpr int kPairRows = 128;
// Cache slots per CTA of the pair kernel. A fifth slot (room made by holding all of Q in
// TMEM and single-buffering S) measured no faster than four on B200: the kernel is bound by
// its per-tile hand-offs, not by the bytes in flight.
constexpr int kPairMaxSlots = 4;
size_t decode_pair_smem_bytes(int r, int rope_half, int nslot);
// Clusters of two that can be resident at once with `smem` bytes each (0 if unknown).
int decode_pair_max_clusters(size_t smem);
cudaError_t launch_decode_pair(const DecodeParams& p, dim3 grid, size_t smem,
                               cudaStream_t stream);

// Merge of the per-piece partials of units cut between CTAs (log-sum-exp identity).
struct CombineParams {
  const uint16_t* part_o;    // bf16
  const float* part_lse;
  const int32_t* unit_start;
  const int32_t* range_len;
  const int32_t* seq_lens;
  uint16_t* o_latent;
  float* lse;
  int32_t q_len, max_seq_len, max_pages, qH, r, ncol, col_groups, units;
  int32_t vgrid;             // work ranges the decode used (pieces per unit ~ vgrid / units)
  int32_t sms;               // SMs of the device (sizes the row-merge grid)
  // optional: bytes the next kernel of the step reads (the up-projection's weights), brought
  // into L2 by the merge blocks before they wait for the decode grid (null: none)
  const void* l2_prefetch;
  int64_t l2_prefetch_bytes;
};
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

}  // namespace mla
