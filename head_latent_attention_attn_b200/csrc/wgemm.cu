// wgemm.cu - per-head weight GEMM on tcgen05 for mla_absorb_q and mla_out_up.
//
// Both steps are "one small weight matrix per head times a few activation rows":
//   absorb:  q_c[n, h, :]  = W_UK[h]^T q_nope[n, h, :]   (W_UK[h] stored [d_n][r])
//   out_up:  o[n, h, :]    = W_UV[h]   o_latent[n, h, :] (W_UV[h] stored [d_v][r])
// The weights dominate the bytes, so the output features are the UMMA M dimension
// (128 per work item) and the activation rows the N dimension; D[m, n] lives in TMEM with
// one output feature per lane.
//
// The grid is persistent: one CTA per SM walks the work items (head, 128-feature tile,
// row tile) with a stride of the grid size. Per item the weight tile is only 16-128 KB,
// so a CTA per item would spend most of its life on setup and on the first load's
// latency; here the TMA ring runs on across items and the whole K of an item (up to 8
// stages) can be in flight at once. Warp 0 issues the TMA loads, warp 1 the UMMAs into
// one of two TMEM accumulators, and warps 2-5 (one per TMEM sub-partition) drain the
// other accumulator, so an item's epilogue overlaps the next item's loads and UMMAs. For
// the absorb step the epilogue warps first write q_ext's rotary slots (and, in the one-call
// decode step, the new tokens' cache rows).
#include "append.cuh"
#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

namespace {
constexpr int kWgThreads = 192;        // warp 0 TMA, warp 1 UMMA, warps 2-5 epilogue
constexpr int kWgEpiThreads = 128;
constexpr int kWgABytes = 128 * 128;   // 128 x 64 bf16 weight tile (two 64x64 boxes for W_UK)

// Shared memory: the TMA stages, 256 bytes of barriers, two epilogue staging tiles of
// [NR rows][128 features] bf16, 1 KB alignment slack.
template <int NR>
struct WgLayout {
  static constexpr int kB = NR * 128;                 // NR rows x 64 bf16
  static constexpr int kStage = kWgABytes + kB;
  static constexpr int kEpi = NR * 128 * 2;           // one staging tile
  static constexpr int kFit = (227 * 1024 - 256 - 2 * kEpi - 1024) / kStage;
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kBars = kStage * kStages;      // barriers after the stages
  static constexpr int kEpiOff = kBars + 256;
  static constexpr int kTotal = kEpiOff + 2 * kEpi + 1024;
};

MLA_DEVICE uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Work item `it` -> (head, first output feature, first activation row).
struct WgItem {
  int h, m0, n0;
  MLA_DEVICE WgItem(int it, int n_mt, int n_nt, int nr) {
    const int nt = it % n_nt;
    const int hm = it / n_nt;
    h = hm / n_mt;
    m0 = (hm % n_mt) * 128;
    n0 = nt * nr;
  }
};

// One rotary chunk: outputs j..j+3 and j+half..j+half+3 of the (n, h, group) slice `seg`
// (c = j / 4). Split into an address/load step and a compute/store step so that a thread
// can issue the loads of several chunks before it waits on any of them.
struct RopeChunk {
  uint16_t* out;
  uint2 x0, x1;
  float4 cv, sv;
  bool own, live;
};

MLA_DEVICE void rope_chunk_load(const WGemmParams& p, int64_t s, int64_t chunks, int cpp,
                                RopeChunk& k) {
  k.live = s < chunks;
  k.own = false;
  if (!k.live) return;
  const int G = p.groups, dr = p.rope_dim, half = dr / 2;
  const int c = int(s % cpp);
  const int64_t seg = s / cpp;
  const int g = int(seg % G);
  const int64_t nh = seg / G;
  const int h = int(nh % p.heads);
  const int n = int(nh / p.heads);
  const int j = 4 * c;
  k.out = p.out + int64_t(n) * p.out_row_stride + int64_t(h) * p.out_head_stride + p.M +
          int64_t(g) * dr + j;
  k.own = g == h / (p.heads / G);
  if (k.own) {
    const uint16_t* q = p.q_pe + (int64_t(n) * p.heads + h) * dr + j;
    const int64_t ci = (int64_t(n) * G + g) * half + j;
    k.x0 = __ldg(reinterpret_cast<const uint2*>(q));
    k.x1 = __ldg(reinterpret_cast<const uint2*>(q + half));
    k.cv = __ldg(reinterpret_cast<const float4*>(p.rope_cos + ci));
    k.sv = __ldg(reinterpret_cast<const float4*>(p.rope_sin + ci));
  }
}

MLA_DEVICE void rope_chunk_store(const WGemmParams& p, const RopeChunk& k) {
  if (!k.live) return;
  const int half = p.rope_dim / 2;
  uint2 lo = make_uint2(0u, 0u), hi = make_uint2(0u, 0u);
  if (k.own) {
    const float a[4] = {__uint_as_float(k.x0.x << 16), __uint_as_float(k.x0.x & 0xFFFF0000u),
                        __uint_as_float(k.x0.y << 16), __uint_as_float(k.x0.y & 0xFFFF0000u)};
    const float b[4] = {__uint_as_float(k.x1.x << 16), __uint_as_float(k.x1.x & 0xFFFF0000u),
                        __uint_as_float(k.x1.y << 16), __uint_as_float(k.x1.y & 0xFFFF0000u)};
    const float cc[4] = {k.cv.x, k.cv.y, k.cv.z, k.cv.w};
    const float ss[4] = {k.sv.x, k.sv.y, k.sv.z, k.sv.w};
    uint16_t y0[4], y1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      y0[i] = f32_to_bf16_rne(__fsub_rn(__fmul_rn(a[i], cc[i]), __fmul_rn(b[i], ss[i])));
      y1[i] = f32_to_bf16_rne(__fadd_rn(__fmul_rn(b[i], cc[i]), __fmul_rn(a[i], ss[i])));
    }
    lo = make_uint2(uint32_t(y0[0]) | (uint32_t(y0[1]) << 16),
                    uint32_t(y0[2]) | (uint32_t(y0[3]) << 16));
    hi = make_uint2(uint32_t(y1[0]) | (uint32_t(y1[1]) << 16),
                    uint32_t(y1[2]) | (uint32_t(y1[3]) << 16));
  }
  *reinterpret_cast<uint2*>(k.out) = lo;
  *reinterpret_cast<uint2*>(k.out + half) = hi;
}

// q_ext's rotary slots [r, r + G d_r) of every (row n, head h): RoPE(q_pe[n, h]) in the
// slice of h's key group, zeros in the other groups' slices. The work is cut into chunks
// of four rotation pairs (outputs j..j+3 and j+half..j+half+3 of one (n, h, group) slice)
// spread over a grid-stride loop, four chunks a thread per step with all their loads issued
// first; a chunk is two 8-byte loads of q_pe, a 16-byte load each of cos and sin, and two
// 8-byte stores. When the half width is not a multiple of 4 or the inputs lack that
// alignment (the host checks both), a slice is one scalar step.
MLA_DEVICE void write_rope_slots(const WGemmParams& p, int tid, int nthreads) {
  const int G = p.groups, dr = p.rope_dim, half = dr / 2;
  if (p.rope_vec != 0) {   // host-checked: alignment and half % 4 == 0
    const int cpp = half / 4;                       // chunks per (n, h, group) slice
    const int64_t chunks = int64_t(p.rows) * p.heads * G * cpp;
    constexpr int kBatch = 4;
    for (int64_t s0 = tid; s0 < chunks; s0 += int64_t(kBatch) * nthreads) {
      RopeChunk k[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) rope_chunk_load(p, s0 + int64_t(u) * nthreads, chunks, cpp, k[u]);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) rope_chunk_store(p, k[u]);
    }
    return;
  }
  const int64_t segs = int64_t(p.rows) * p.heads * G;
  for (int64_t s = tid; s < segs; s += nthreads) {
    const int g = int(s % G);
    const int64_t nh = s / G;
    const int h = int(nh % p.heads);
    const int n = int(nh / p.heads);
    uint16_t* out = p.out + int64_t(n) * p.out_row_stride + int64_t(h) * p.out_head_stride + p.M +
                    int64_t(g) * dr;
    if (g != h / (p.heads / G)) {
      for (int j = 0; j < dr; ++j) out[j] = 0;
      continue;
    }
    const uint16_t* q = p.q_pe + (int64_t(n) * p.heads + h) * dr;
    const float* cs = p.rope_cos + (int64_t(n) * G + g) * half;
    const float* sn = p.rope_sin + (int64_t(n) * G + g) * half;
    for (int j = 0; j < half; ++j) {
      const float x0 = bf16_bits_to_f32(__ldg(q + j));
      const float x1 = bf16_bits_to_f32(__ldg(q + j + half));
      const float cj = __ldg(cs + j);
      const float sj = __ldg(sn + j);
      out[j] = f32_to_bf16_rne(__fsub_rn(__fmul_rn(x0, cj), __fmul_rn(x1, sj)));
      out[j + half] = f32_to_bf16_rne(__fadd_rn(__fmul_rn(x1, cj), __fmul_rn(x0, sj)));
    }
  }
}
}  // namespace

// Epilogue of absorb / out_up for one item, run by the four epilogue warps: the
// accumulator (output feature m0 + lane of each TMEM lane, one column per activation row)
// plus the bias is rounded to bf16 into a [NR rows][128 features] staging tile (two
// tiles, used by alternate items), the accumulator is handed back, and one thread stores
// the tile with the TMA (rows out_row_stride apart, columns past M and rows past `rows`
// clipped). Before a tile is written again the store that read it two items earlier has
// finished reading it (bulk_wait_read<1> after each store, then the closing barrier).
// Without the tensor map (strides that are no multiple of 16 bytes) the threads copy the
// tile element by element. All four warps pass both named barriers whatever their
// accumulator wait returned (`ok`); a failed wait leaves the CTA's abort flag set, and
// then the tile is not written.
template <int NR>
MLA_DEVICE void plain_epilogue(const WGemmParams& p, const WgItem& w, int buf, uint32_t tmem,
                               int sp, int lane, uint16_t* stage, uint64_t* acc_empty, bool ok,
                               volatile int* abort_flag) {
  const int m_loc = sp * 32 + lane;
  const int m = w.m0 + m_loc;                  // output feature of this thread's TMEM lane
  if (ok) {
    const float bias = (p.bias != nullptr && m < p.M)
                           ? bf16_bits_to_f32(p.bias[int64_t(w.h) * p.M + m]) : 0.0f;
    // Not unrolled: the code runs once per item with a cold instruction cache (the decode
    // kernel runs between these launches).
#pragma unroll 1
    for (int c0 = 0; c0 < NR; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + (uint32_t(sp * 32) << 16) + uint32_t(buf * NR + c0), v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) stage[(c0 + j) * 128 + m_loc] = cvt_bf16(v[j] + bias);
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);
  if (p.tma_out != 0) {
    fence_proxy_async_smem();                  // the tile's writes, seen by the TMA
    named_bar_sync(1, kWgEpiThreads);          // the staging tile is complete
    if (m_loc == 0) {
      if (*abort_flag == 0) {
        tma_store_3d(&p.tm_out, stage, w.m0, w.h, w.n0);
        bulk_commit();
      }
      bulk_wait_read<1>();                     // the other tile's store has read it
    }
    named_bar_sync(1, kWgEpiThreads);
    return;
  }
  named_bar_sync(1, kWgEpiThreads);            // the staging tile is complete
  if (*abort_flag == 0) {
    const int nrows = min(NR, p.rows - w.n0);
    const int mt = min(128, p.M - w.m0);       // features of this tile
    uint16_t* out = p.out + int64_t(w.n0) * p.out_row_stride + int64_t(w.h) * p.out_head_stride +
                    w.m0;
    for (int idx = m_loc; idx < nrows * mt; idx += kWgEpiThreads) {
      const int n = idx / mt, c = idx - (idx / mt) * mt;
      out[int64_t(n) * p.out_row_stride + c] = stage[n * 128 + c];
    }
  }
  named_bar_sync(1, kWgEpiThreads);            // the staging tile may be reused
}

template <int NR>
__global__ void __launch_bounds__(kWgThreads, 1) wgemm_kernel(const __grid_constant__ WGemmParams p) {
  using Lay = WgLayout<NR>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Lay::kBars);   // [S] stage landed
  uint64_t* empty = full + S;                                         // [S] stage consumed
  uint64_t* acc_full = empty + S;                                     // [2] accumulator ready
  uint64_t* acc_empty = acc_full + 2;                                 // [2] accumulator drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_mt = (p.M + 127) / 128;
  const int n_nt = (p.rows + NR - 1) / NR;
  const int nk = (p.K + 63) / 64;
  const int items = n_mt * p.heads * n_nt;
  constexpr uint32_t kCols = 2 * NR < 32 ? 32 : 2 * NR;   // two accumulators of NR columns
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);                    // the four epilogue warps
    }
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
    // ======================= TMA producer: weight and activation tiles ===================
    if (elect_one()) {
      prefetch_tensormap(&p.tm_w);
      prefetch_tensormap(&p.tm_x);
      if (p.tma_out) prefetch_tensormap(&p.tm_out);
      // The weights are no kernel's output here: warm L2 with this CTA's weight tiles while
      // the previous kernel may still run (an L2 prefetch is coherent with any writer).
      for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const WgItem w(it, n_mt, n_nt, NR);
        for (int kb = 0; kb < nk; ++kb) {
          if (p.a_mn) {
            tma_prefetch_l2_3d(&p.tm_w, w.m0, kb * 64, w.h);
            tma_prefetch_l2_3d(&p.tm_w, w.m0 + 64, kb * 64, w.h);
          } else {
            tma_prefetch_l2_3d(&p.tm_w, kb * 64, w.m0, w.h);
          }
        }
      }
    }
    __syncwarp();
    grid_dep_wait();
    grid_dep_launch();
    if (elect_one()) {
      SlotRing ring(S);
      int g = 0;   // stages issued
      bool ok = true;
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
        const WgItem w(it, n_mt, n_nt, NR);
        for (int kb = 0; kb < nk; ++kb, ++g, ring.next()) {
          if (g >= S && !mbar_wait(&empty[ring.slot], (ring.round - 1) & 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* a = base + ring.slot * Lay::kStage;
          uint8_t* b = a + kWgABytes;
          mbar_arrive_expect_tx(&full[ring.slot], Lay::kStage);
          if (p.a_mn) {
            tma_load_3d(a, &p.tm_w, w.m0, kb * 64, w.h, &full[ring.slot]);
            tma_load_3d(a + 8192, &p.tm_w, w.m0 + 64, kb * 64, w.h, &full[ring.slot]);
          } else {
            tma_load_3d(a, &p.tm_w, kb * 64, w.m0, w.h, &full[ring.slot]);
          }
          tma_load_3d(b, &p.tm_x, kb * 64, w.h, w.n0, &full[ring.slot]);
        }
      }
      // never leave with copies in flight into this CTA's shared memory
      for (int j = (g > S ? g - S : 0); j < g; ++j)
        mbar_wait_bounded(&full[j % S], (j / S) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ UMMA issuer, two accumulators ==========================
    grid_dep_wait();
    grid_dep_launch();
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(128, NR, p.a_mn, 0);
      SlotRing ring(S);
      bool ok = true;
      int li = 0;   // items of this CTA so far
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x, ++li) {
        const WgItem w(it, n_mt, n_nt, NR);
        const int buf = li & 1;
        // the epilogue has drained this accumulator (item li - 2)
        if (li >= 2 && !mbar_wait(&acc_empty[buf], ((li >> 1) - 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(buf * NR);
        for (int kb = 0; kb < nk; ++kb, ring.next()) {
          if (!mbar_wait(&full[ring.slot], ring.round & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(base + ring.slot * Lay::kStage);
          const uint32_t b = a + kWgABytes;
          const int rem = p.K - kb * 64;
          const int nkk = rem >= 64 ? 4 : (rem + 15) / 16;
          for (int kk = 0; kk < nkk; ++kk) {
            const uint64_t ad = p.a_mn ? make_sdesc(a + kk * 2048, 8192, 1024, kSw128)
                                       : make_sdesc(a + kk * 32, 16, 1024, kSw128);
            const uint64_t bd = make_sdesc(b + kk * 32, 16, 1024, kSw128);
            umma_bf16(d, ad, bd, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
          }
          umma_commit(&empty[ring.slot]);
        }
        if (ok) umma_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else {
    // ============== epilogue warps 2-5: warp w reaches TMEM lanes 32 (w % 4) .. ==========
    grid_dep_wait();
    grid_dep_launch();
    const int sp = warp & 3;
    {
      // new tokens' cache rows (one warp per token) while the first accumulator fills; dealt
      // from the last CTA down, since the items are dealt from the first CTA up and the last
      // CTAs may hold one item fewer
      const int64_t ntok = int64_t(p.app.batch) * p.app.n_new;
      for (int64_t gw = int64_t(gridDim.x - 1 - blockIdx.x) * 4 + (warp - 2); gw < ntok;
           gw += int64_t(gridDim.x) * 4)
        append_token(p.app, gw, lane);
    }
    if (p.q_pe != nullptr && p.rope_dim > 0)
      write_rope_slots(p, int(blockIdx.x) * kWgEpiThreads + int(threadIdx.x) - 64,
                       int(gridDim.x) * kWgEpiThreads);
    int li = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++li) {
      const WgItem w(it, n_mt, n_nt, NR);
      const int buf = li & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (li >> 1) & 1, wc));
      tc_fence_after();
      plain_epilogue<NR>(p, w, buf, tmem, sp, lane,
                         reinterpret_cast<uint16_t*>(base + Lay::kEpiOff + (li & 1) * Lay::kEpi),
                         &acc_empty[buf], ok, abort_flag);
    }
    // the last tiles' stores have written global memory before the CTA leaves
    if (p.tma_out != 0 && sp == 0 && lane == 0) bulk_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kCols);
}

template <int NR>
static cudaError_t launch_wgemm_nr(const WGemmParams& p, int max_ctas, cudaStream_t stream) {
  const int smem = WgLayout<NR>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(wgemm_kernel<NR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t items = int64_t((p.M + 127) / 128) * p.heads * ((p.rows + NR - 1) / NR);
  const int grid = int(items < max_ctas ? items : max_ctas);
  return launch_pdl(wgemm_kernel<NR>, dim3(grid), dim3(kWgThreads), size_t(smem), stream, 1, p);
}

cudaError_t launch_wgemm(const WGemmParams& p, int nr, int max_ctas, cudaStream_t stream) {
  if (max_ctas <= 0) return cudaErrorInvalidValue;
  switch (nr) {
    case 16: return launch_wgemm_nr<16>(p, max_ctas, stream);
    case 32: return launch_wgemm_nr<32>(p, max_ctas, stream);
    case 64: return launch_wgemm_nr<64>(p, max_ctas, stream);
    case 128: return launch_wgemm_nr<128>(p, max_ctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
