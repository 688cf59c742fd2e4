// oproj.cu - mla_out_proj: the value up-projection and the output projection of the
// DeepSeek-V2 page's "Matrix absorption" section, einsums (5) and (6), in one kernel:
//   stage A, per head h:              o[n, h, :] = W_UV[h] o_[n, h, :] (+ up_v bias)   K = r
//   stage B, per 128 model features:  u[n, k]    = sum_(h, d) W_o[k, h d_v + d] o[n, h, d]
//                                                  (+ bias)                          K = H d_v
// Both are weight-streaming GEMMs on tcgen05 with the output features on UMMA M and the n
// activation rows on N (like wgemm.cu). Stage B reads stage A's output, so the kernel is
// persistent and co-resident (a cooperative launch): every CTA takes its stage-A items
// first; a stage-B item waits, in its TMA producer only, for per-head completion counters
// that the stage-A epilogues release (polled with one round of relaxed loads, then one
// acquire fence), and streams its W_o tiles as soon as those heads are done. Stage B's K is cut into S splits so that its items fill the GPU in about one wave
// (W_o is the bulk of the bytes: 168 MB at the DeepSeek-V2 shape, o only 2 MB and L2
// resident); each split stores an fp32 partial, and the last split of a tile to finish (a
// counter per tile) adds the S partials in a fixed order and writes u in bf16, so the
// result does not depend on which split finished first. The counters are cleared again by
// the kernel (the last CTA to leave resets the per-head counters), so a zeroed workspace
// stays reusable.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 UMMA issuer (two TMEM accumulators),
// warps 2-5 epilogue, one per TMEM sub-partition (output feature = TMEM lane).
#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

namespace {
constexpr int kOpThreads = 192;
constexpr int kOpEpi = 128;
constexpr int kOpABytes = 128 * 128;                 // 128 x 64 bf16 weight tile

template <int NR>
struct OpLayout {
  static constexpr int kB = NR * 128;                // NR rows x 64 bf16
  static constexpr int kStage = kOpABytes + kB;
  static constexpr int kFit = (192 * 1024) / kStage;
  static constexpr int kStages = kFit < 8 ? kFit : 8;
  static constexpr int kBars = kStage * kStages;
  static constexpr int kTotal = kBars + 256 + 1024;
};

MLA_DEVICE uint8_t* op_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

MLA_DEVICE int ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MLA_DEVICE void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
MLA_DEVICE void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Item `it` of the kernel: stage A items first (head, feature tile, row tile), then stage B
// items (model-feature tile, K split, row tile).
struct OpItem {
  bool b;              // stage B
  int h, m0, n0;       // A: head; both: first output feature and first activation row
  int s, tile;         // B: split and (feature tile, row tile) index of the reduction counter
  int k0, nk;          // first K element and number of 64-element K blocks
  MLA_DEVICE OpItem(const OProjParams& p, int it, int NR) {
    const int n_nt = (p.rows + NR - 1) / NR;
    const int mtA = (p.dv + 127) / 128;
    const int nA = p.H * mtA * n_nt;
    if (it < nA) {
      b = false;
      const int nt = it % n_nt, hm = it / n_nt;
      h = hm / mtA;
      m0 = (hm % mtA) * 128;
      n0 = nt * NR;
      s = tile = 0;
      k0 = 0;
      nk = (p.r + 63) / 64;
    } else {
      b = true;
      const int j = it - nA;
      const int nt = j % n_nt, rest = j / n_nt;
      s = rest % p.splits;
      const int mt = rest / p.splits;
      h = 0;
      m0 = mt * 128;
      n0 = nt * NR;
      tile = mt * n_nt + nt;
      const int h0 = s * p.H / p.splits, h1 = (s + 1) * p.H / p.splits;
      k0 = h0 * p.dv;
      nk = (h1 - h0) * p.dv / 64;       // d_v % 64 == 0 (host-checked)
    }
  }
};
}  // namespace

template <int NR>
__global__ void __launch_bounds__(kOpThreads, 1) oproj_kernel(const __grid_constant__ OProjParams p) {
  using Lay = OpLayout<NR>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = op_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Lay::kBars);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_nt = (p.rows + NR - 1) / NR;
  const int mtA = (p.dv + 127) / 128;
  const int items = p.H * mtA * n_nt + ((p.hidden + 127) / 128) * p.splits * n_nt;
  const int headA_target = mtA * n_nt;              // stage-A items per head
  constexpr uint32_t kCols = 2 * NR < 32 ? 32 : 2 * NR;
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    *last_flag = 0;
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
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ======================= TMA producer =======================================
    if (elect_one()) {
      prefetch_tensormap(&p.tm_wuv);
      prefetch_tensormap(&p.tm_ol);
      prefetch_tensormap(&p.tm_wo);
      prefetch_tensormap(&p.tm_o);
      SlotRing ring(S);
      int g = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x) {
        const OpItem w(p, it, NR);
        bool need = w.b;                            // stage B: wait for its heads once
        for (int kb = 0; kb < w.nk; ++kb, ++g, ring.next()) {
          if (g >= S && !mbar_wait(&empty[ring.slot], (ring.round - 1) & 1, wc)) {
            ok = false;
            break;
          }
          uint8_t* a = base + ring.slot * Lay::kStage;
          uint8_t* bb = a + kOpABytes;
          mbar_arrive_expect_tx(&full[ring.slot], Lay::kStage);
          if (!w.b) {
            tma_load_3d(a, &p.tm_wuv, kb * 64, w.m0, w.h, &full[ring.slot]);
            tma_load_3d(bb, &p.tm_ol, kb * 64, w.h, w.n0, &full[ring.slot]);
            continue;
          }
          tma_load_2d(a, &p.tm_wo, w.k0 + kb * 64, w.m0, &full[ring.slot]);
          if (need) {
            // o of this split's heads is written by stage-A epilogues of any CTA. Each pass
            // reads every head's counter with independent relaxed loads (one L2 round trip
            // for all of them, not one per head); once all are complete, one acquire fence
            // orders the o loads below after the epilogues' release.
            const int h0 = w.s * p.H / p.splits, h1 = (w.s + 1) * p.H / p.splits;
            const uint64_t t0 = globaltimer_ns();
            while (true) {
              bool all = true;
              for (int h = h0; h < h1; ++h) all &= ld_relaxed(p.head_done + h) >= headA_target;
              if (all) break;
              __nanosleep(128);
              if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                if (p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_TIMEOUT);
                ok = false;
                break;
              }
            }
            fence_acq_rel_gpu();
            fence_proxy_async_global();
            need = false;
          }
          // after a failed wait the stage still completes (the data is not used)
          tma_load_2d(bb, &p.tm_o, w.k0 + kb * 64, w.n0, &full[ring.slot]);
          if (!ok) {
            ++g;
            ring.next();
            break;
          }
        }
      }
      for (int j = (g > S ? g - S : 0); j < g; ++j)
        mbar_wait_bounded(&full[j % S], (j / S) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================= UMMA issuer ========================================
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(128, NR, 0, 0);
      SlotRing ring(S);
      bool ok = true;
      int li = 0;
      for (int it = blockIdx.x; ok && it < items; it += gridDim.x, ++li) {
        const OpItem w(p, it, NR);
        const int buf = li & 1;
        if (li >= 2 && !mbar_wait(&acc_empty[buf], ((li >> 1) - 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(buf * NR);
        const int kmax = w.b ? w.nk * 64 : p.r;
        for (int kb = 0; kb < w.nk; ++kb, ring.next()) {
          if (!mbar_wait(&full[ring.slot], ring.round & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(base + ring.slot * Lay::kStage);
          const uint32_t bb = a + kOpABytes;
          const int rem = kmax - kb * 64;
          const int nkk = rem >= 64 ? 4 : (rem + 15) / 16;
          for (int kk = 0; kk < nkk; ++kk)
            umma_bf16(d, make_sdesc(a + kk * 32, 16, 1024, kSw128),
                      make_sdesc(bb + kk * 32, 16, 1024, kSw128), idesc, (kb | kk) != 0);
          umma_commit(&empty[ring.slot]);
        }
        if (ok) umma_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else {
    // ======================= epilogue warps 2-5 ================================
    // Every named barrier below is passed by all four warps whatever their waits returned;
    // a failed wait leaves the abort flag set and then nothing further is written.
    const int sp = warp & 3;
    const int lane_m = sp * 32 + lane;
    const bool leader = (warp == 2 && lane == 0);
    int li = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++li) {
      const OpItem w(p, it, NR);
      const int buf = li & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (li >> 1) & 1, wc));
      tc_fence_after();
      const int nrows = min(NR, p.rows - w.n0);
      const int m = w.m0 + lane_m;
      if (ok && !w.b) {
        // stage A: o[n, h, m] in bf16 (+ up_v bias)
        const bool live = m < p.dv;
        const float bias = (p.bias_v != nullptr && live)
                               ? bf16_bits_to_f32(p.bias_v[int64_t(w.h) * p.dv + m]) : 0.0f;
        uint16_t* out = p.o + (int64_t(w.n0) * p.H + w.h) * p.dv + m;
        const int64_t rs = int64_t(p.H) * p.dv;
#pragma unroll 1
        for (int c0 = 0; c0 < NR; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + (uint32_t(sp * 32) << 16) + uint32_t(buf * NR + c0), v);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < nrows) out[int64_t(c0 + j) * rs] = f32_to_bf16_rne(v[j] + bias);
          }
        }
        // visible to stage B's TMA loads in any CTA before the head counter moves
        fence_proxy_async_global();
        __threadfence();
      } else if (ok) {
        // stage B: fp32 partial of split s for features m of the row tile
        const bool live = m < p.hidden;
        float* dst = p.part + (int64_t(w.s) * p.rows + w.n0) * p.hidden + m;
#pragma unroll 1
        for (int c0 = 0; c0 < NR; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + (uint32_t(sp * 32) << 16) + uint32_t(buf * NR + c0), v);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < nrows) dst[int64_t(c0 + j) * p.hidden] = v[j];
          }
        }
        __threadfence();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      named_bar_sync(1, kOpEpi);
      if (leader && *abort_flag == 0) {
        if (!w.b) {
          atomicAdd(p.head_done + w.h, 1);   // after the fences above: a release of this tile
        } else {
          const int old = atomicAdd(p.tile_done + w.tile, 1);
          *last_flag = (old == p.splits - 1) ? 1 : 0;
        }
      }
      named_bar_sync(1, kOpEpi);
      if (w.b && *last_flag != 0 && *abort_flag == 0) {
        // the last split of this tile: u = sum of the S partials in split order (+ bias),
        // four consecutive features per thread and step, the loads of several rows in flight
        __threadfence();
        const int nq = 32;                            // 4-feature groups of the 128-feature tile
        const int64_t ps = int64_t(p.rows) * p.hidden;
#pragma unroll 4
        for (int idx = lane_m; idx < nrows * nq; idx += kOpEpi) {
          const int n = idx / nq, k = w.m0 + 4 * (idx - (idx / nq) * nq);
          if (k >= p.hidden) continue;                // hidden % 8 == 0: groups are whole
          const int64_t off = int64_t(w.n0 + n) * p.hidden + k;
          float4 acc = __ldcg(reinterpret_cast<const float4*>(p.part + off));
          for (int s = 1; s < p.splits; ++s) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(p.part + s * ps + off));
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
          if (p.bias_o != nullptr) {
            acc.x += bf16_bits_to_f32(p.bias_o[k]);
            acc.y += bf16_bits_to_f32(p.bias_o[k + 1]);
            acc.z += bf16_bits_to_f32(p.bias_o[k + 2]);
            acc.w += bf16_bits_to_f32(p.bias_o[k + 3]);
          }
          *reinterpret_cast<uint2*>(p.u + off) =
              make_uint2(cvt_bf16x2(acc.x, acc.y), cvt_bf16x2(acc.z, acc.w));
        }
        if (leader) p.tile_done[w.tile] = 0;
      }
      named_bar_sync(1, kOpEpi);
      if (leader) *last_flag = 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kCols);
  // the last CTA to leave clears the per-head counters for the next call
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(p.cta_done, 1);
    if (old == int(gridDim.x) - 1) {
      for (int h = 0; h < p.H; ++h) p.head_done[h] = 0;
      __threadfence();
      *p.cta_done = 0;
    }
  }
}

size_t oproj_smem_bytes(int nr) {
  switch (nr) {
    case 16: return OpLayout<16>::kTotal;
    case 32: return OpLayout<32>::kTotal;
    case 64: return OpLayout<64>::kTotal;
    default: return OpLayout<128>::kTotal;
  }
}

template <int NR>
static cudaError_t launch_oproj_nr(const OProjParams& p, int grid, cudaStream_t stream) {
  const int smem = OpLayout<NR>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(oproj_kernel<NR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // every CTA must be resident at once (stage B waits for stage A of other CTAs)
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, oproj_kernel<NR>, kOpThreads, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (per_sm < 1 || grid > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kOpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, oproj_kernel<NR>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_oproj(const OProjParams& p, int nr, int grid, cudaStream_t stream) {
  switch (nr) {
    case 16: return launch_oproj_nr<16>(p, grid, stream);
    case 32: return launch_oproj_nr<32>(p, grid, stream);
    case 64: return launch_oproj_nr<64>(p, grid, stream);
    case 128: return launch_oproj_nr<128>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
