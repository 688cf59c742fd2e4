// down_kv.cu - mla_down_kv_append: [c_kv ; k_r] = W_DKV x for new tokens, written straight
// into the paged cache (kv_a_proj_with_mqa of the DeepSeek-V2 page, eq. (41); down_kv and
// k_r_proj of the MLAfication page).
//
// The output features are the UMMA M dimension: ceil(r/128) latent tiles of 128 and one
// rotary tile starting at feature r (every rotation pair of every group then sits in one
// tile); the token rows are the N dimension (NR per tile). The weights are the bytes, and
// the model width K is long (5120 at the DeepSeek-V2 shape) while there are only a few
// tiles, so K is split across a cluster of C CTAs:
//   * CTA k of the cluster accumulates K blocks [k nk / C, (k + 1) nk / C) of its tile in
//     TMEM (warp 0 TMA ring, warp 1 UMMA issuer), then warps 2-5 copy the fp32 partial into
//     the CTA's shared memory (the TMA stages are free by then);
//   * after a cluster barrier, CTA k reduces rows [k NR / C, (k + 1) NR / C) of the tile over
//     the C partials, read through distributed shared memory in rank order (the sum does not
//     depend on timing), rounds them to bf16 and writes those tokens' cache rows exactly as
//     mla_cache_append does (the rotary features rotated in fp32 with separately rounded
//     products and sums, from the rounded values), and kv_out if given;
//   * a second cluster barrier keeps every CTA's shared memory alive until all reads of it
//     are done.
// No global atomics and no workspace. Every wait is bounded; a CTA whose wait gave up still
// passes both cluster barriers (with the abort flag set, nothing is written).
#include <algorithm>

#include "kernels.h"
#include "ptx.cuh"

namespace mla {

namespace {

constexpr int kDkvThreads = 192;      // warp 0 TMA, warp 1 UMMA, warps 2-5 epilogue
constexpr int kDkvABytes = 128 * 128; // 128 features x 64 K (bf16)
constexpr int kDkvMaxSplits = 16;     // cluster size limit (16: non-portable, opted in)

template <int NR>
struct DkvLayout {
  static constexpr int kB = NR * 128;                       // NR rows x 64 K (bf16)
  static constexpr int kStage = kDkvABytes + kB;
  static constexpr int kPart = NR * 128 * 4;                // fp32 partial [NR][128]
  static constexpr int kStageFit = (200 * 1024) / kStage;
  static constexpr int kStages = kStageFit < 8 ? kStageFit : 8;
  static constexpr int kArea = kStage * kStages;             // stages; later partial + rows
  static constexpr int kBars = kArea;
  static constexpr int kSlots = kBars + 256;                 // int64 cache row per token
  static constexpr int kTotal = kSlots + NR * 8 + 1024;
  static_assert(kPart + NR * 128 * 2 <= kArea, "partial and row tile must fit the stages");
};

MLA_DEVICE uint8_t* dkv_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

MLA_DEVICE float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Physical cache row of token `row` (token t of sequence b), or -1 when its position or page
// is out of range.
MLA_DEVICE int64_t dkv_slot(const DkvParams& p, int row) {
  const int b = row / p.n_new;
  const int t = row - b * p.n_new;
  const int64_t pos = int64_t(p.start_pos[b]) + t;
  const int64_t lp = pos >= 0 ? pos / p.page_size : -1;
  if (pos < 0 || lp >= p.max_pages) return -1;
  const int32_t page = p.block_table[int64_t(b) * p.max_pages + lp];
  if (page < 0 || page >= p.num_pages) return -1;
  return int64_t(page) * p.page_size + pos % p.page_size;
}

}  // namespace

template <int NR>
__global__ void __launch_bounds__(kDkvThreads, 1)
    down_kv_kernel(const __grid_constant__ DkvParams p) {
  using Lay = DkvLayout<NR>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = dkv_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Lay::kBars);   // [S]
  uint64_t* empty = full + S;                                         // [S]
  uint64_t* acc_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* part = reinterpret_cast<float*>(base);                       // [NR][128] after UMMAs
  uint16_t* rowt = reinterpret_cast<uint16_t*>(base + Lay::kPart);    // [NR][128] bf16
  int64_t* slots = reinterpret_cast<int64_t*>(base + Lay::kSlots);    // [NR] cache rows

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.splits;
  const int k = int(cluster_ctarank());                               // split of this CTA
  const int tile = int(blockIdx.x) / C;
  const int mt = tile / p.n_nt, nt = tile - (tile / p.n_nt) * p.n_nt;
  const int m0 = mt < p.lat_tiles ? mt * 128 : p.r;                   // first output feature
  const int n0 = nt * NR;
  const int nk = (p.K + 63) / 64;
  const int kb0 = k * nk / C, kb1 = (k + 1) * nk / C;
  constexpr uint32_t kCols = NR < 32 ? 32 : NR;
  const WaitCtx wc{abort_flag, p.dev_error};
  const int rpc = (NR + C - 1) / C;                    // tokens reduced by each CTA
  const int r_lo = min(NR, k * rpc), r_hi = min(NR, r_lo + rpc);
  const int nrows_tile = min(NR, p.rows - n0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ============================== TMA producer ====================================
    if (elect_one()) {
      prefetch_tensormap(&p.tm_w);
      prefetch_tensormap(&p.tm_x);
      // the weights are no kernel's output: warm L2 while the previous kernel may still run
      for (int kb = kb0; kb < kb1; ++kb) tma_prefetch_l2_2d(&p.tm_w, kb * 64, m0);
    }
    __syncwarp();
    grid_dep_wait();
    grid_dep_launch();
    if (elect_one()) {
      int g = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int slot = g % S;
        if (g >= S && !mbar_wait(&empty[slot], ((g / S) - 1) & 1, wc)) break;
        uint8_t* a = base + slot * Lay::kStage;
        mbar_arrive_expect_tx(&full[slot], Lay::kStage);
        tma_load_2d(a, &p.tm_w, kb * 64, m0, &full[slot]);
        tma_load_2d(a + kDkvABytes, &p.tm_x, kb * 64, n0, &full[slot]);
      }
      // never leave with copies in flight into this CTA's shared memory
      for (int j = (g > S ? g - S : 0); j < g; ++j)
        mbar_wait_bounded(&full[j % S], (j / S) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // =============================== UMMA issuer ====================================
    grid_dep_wait();
    grid_dep_launch();
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(128, NR, 0, 0);
      bool ok = true;
      int g = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int slot = g % S;
        if (!mbar_wait(&full[slot], (g / S) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(base + slot * Lay::kStage);
        const uint32_t b = a + kDkvABytes;
        const int rem = p.K - kb * 64;
        const int nkk = rem >= 64 ? 4 : (rem + 15) / 16;
        for (int kk = 0; kk < nkk; ++kk)
          umma_bf16(tmem, make_sdesc(a + kk * 32, 16, 1024, kSw128),
                    make_sdesc(b + kk * 32, 16, 1024, kSw128), idesc,
                    (kb != kb0 || kk != 0) ? 1u : 0u);
        umma_commit(&empty[slot]);
      }
      if (ok) umma_commit(acc_full);
    }
    __syncwarp();
  } else {
    // ================== epilogue warps: this CTA's fp32 partial to shared ===========
    grid_dep_wait();
    grid_dep_launch();
    const int sp = warp & 3;
    const int f = sp * 32 + lane;                       // feature of this thread's TMEM lane
    // the cache rows of this CTA's tokens, looked up while the UMMAs run
    const int et = int(threadIdx.x) - 64;
    if (et < r_hi - r_lo) {
      const int n = r_lo + et;
      int64_t slot = -2;                                // past the batch: nothing to write
      if (n < nrows_tile) {
        slot = dkv_slot(p, n0 + n);
        if (slot < 0 && p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
      }
      slots[n] = slot;
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, wc));
    tc_fence_after();
#pragma unroll 1
    for (int c0 = 0; c0 < NR; c0 += 16) {
      float v[16];
      if (ok) {
        tmem_ld16(tmem + (uint32_t(sp * 32) << 16) + uint32_t(c0), v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) part[(c0 + j) * 128 + f] = v[j];
    }
    tc_fence_before();
  }
  // every CTA's partial is complete and visible to the cluster
  cluster_sync_all();

  // ===== reduction of rows [k NR / C, (k + 1) NR / C) over the C partials, rank order =====
  const int D = p.r + p.groups * p.rope_dim;
  const int f_end = m0 < p.r ? min(m0 + 128, p.r) : D;  // features of this tile: [m0, f_end)
  const uint32_t part_s = smem_u32(part);
  for (int idx = int(threadIdx.x); idx < (r_hi - r_lo) * 32; idx += kDkvThreads) {
    const int n = r_lo + (idx >> 5), q = 4 * (idx & 31);
    const uint32_t off = part_s + uint32_t((n * 128 + q) * 4);
    float4 v[kDkvMaxSplits];
#pragma unroll
    for (int j = 0; j < kDkvMaxSplits; ++j)   // every partial's load in flight at once
      if (j < C) v[j] = ld_cluster_f4(map_to_rank(off, uint32_t(j)));
    float4 acc = v[0];
#pragma unroll
    for (int j = 1; j < kDkvMaxSplits; ++j) {
      if (j < C) {
        acc.x += v[j].x;
        acc.y += v[j].y;
        acc.z += v[j].z;
        acc.w += v[j].w;
      }
    }
    *reinterpret_cast<uint2*>(rowt + n * 128 + q) =
        make_uint2(cvt_bf16x2(acc.x, acc.y), cvt_bf16x2(acc.z, acc.w));
  }
  __syncthreads();

  // ============== cache rows (and kv_out) of this CTA's tokens, from the bf16 tile ========
  if (*abort_flag == 0) {
    for (int n = r_lo + warp; n < r_hi; n += kDkvThreads / 32) {
      if (n >= nrows_tile) break;
      const int row = n0 + n;
      const int64_t slot = slots[n];
      const uint16_t* src = rowt + n * 128;
      if (m0 < p.r) {
        // latent features [m0, f_end), 8 per 16-byte piece (r % 8 == 0)
        for (int c = lane; c < (f_end - m0) / 8; c += 32) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + 8 * c);
          if (p.kv_out) *reinterpret_cast<uint4*>(p.kv_out + int64_t(row) * D + m0 + 8 * c) = v;
          if (slot >= 0) *reinterpret_cast<uint4*>(p.cache + slot * D + m0 + 8 * c) = v;
        }
      } else {
        // rotary features: pair j of group g = (x_j, x_{j + d_r / 2}) of the group's slice
        const int half = p.rope_dim / 2;
        const int pairs = p.groups * half;
        for (int pi = lane; pi < pairs; pi += 32) {
          const int g = pi / half, j = pi - (pi / half) * half;
          const int fo = g * p.rope_dim + j;              // offset within the rotary tile
          const uint16_t b0 = src[fo], b1 = src[fo + half];
          if (p.kv_out) {
            p.kv_out[int64_t(row) * D + p.r + fo] = b0;
            p.kv_out[int64_t(row) * D + p.r + fo + half] = b1;
          }
          if (slot < 0) continue;
          const float x0 = bf16_bits_to_f32(b0), x1 = bf16_bits_to_f32(b1);
          const int64_t ci = (int64_t(row) * p.groups + g) * half + j;
          const float cj = p.rope_cos[ci], sj = p.rope_sin[ci];
          uint16_t* dst = p.cache + slot * D + p.r + fo;
          dst[0] = f32_to_bf16_rne(__fsub_rn(__fmul_rn(x0, cj), __fmul_rn(x1, sj)));
          dst[half] = f32_to_bf16_rne(__fadd_rn(__fmul_rn(x1, cj), __fmul_rn(x0, sj)));
        }
      }
    }
  }
  // no CTA leaves while another may still read its partial
  cluster_sync_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kCols);
}

// Largest cluster size in {16, 8} that can be resident with this kernel's shared memory
// (16 needs the non-portable opt-in), capped at `want`.
template <int NR>
static int down_kv_cluster(int want) {
  const int smem = DkvLayout<NR>::kTotal;
  if (cudaFuncSetAttribute(down_kv_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess ||
      cudaFuncSetAttribute(down_kv_kernel<NR>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                           1) != cudaSuccess)
    return std::min(want, 8);
  for (int c = 16; c > 8; c /= 2) {
    if (want < c) continue;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(c);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(unsigned(c));
    cfg.blockDim = dim3(kDkvThreads);
    cfg.dynamicSmemBytes = size_t(smem);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, down_kv_kernel<NR>, &cfg) == cudaSuccess && n > 0)
      return c;
    (void)cudaGetLastError();
  }
  return std::min(want, 8);
}

template <int NR>
static cudaError_t launch_down_kv_nr(DkvParams p, cudaStream_t stream) {
  const int smem = DkvLayout<NR>::kTotal;
  p.splits = down_kv_cluster<NR>(p.splits);
  const int n_mt = p.lat_tiles + (p.groups * p.rope_dim > 0 ? 1 : 0);
  const int64_t grid = int64_t(n_mt) * p.n_nt * p.splits;
  return launch_pdl(down_kv_kernel<NR>, dim3(unsigned(grid)), dim3(kDkvThreads), size_t(smem),
                    stream, p.splits, p);
}

cudaError_t launch_down_kv(const DkvParams& p, int nr, cudaStream_t stream) {
  switch (nr) {
    case 16: return launch_down_kv_nr<16>(p, stream);
    case 32: return launch_down_kv_nr<32>(p, stream);
    case 64: return launch_down_kv_nr<64>(p, stream);
    case 128: return launch_down_kv_nr<128>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
