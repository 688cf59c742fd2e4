// wgemm.cu - per-head weight GEMM on tcgen05 for mla_absorb_q and mla_out_up.
//
// Both steps are "one small weight matrix per head times a few activation rows":
//   absorb:  q_c[n, h, :]  = W_UK[h]^T q_nope[n, h, :]   (W_UK[h] stored [d_n][r])
//   out_up:  o[n, h, :]    = W_UV[h]   o_latent[n, h, :] (W_UV[h] stored [d_v][r])
// The weights dominate the bytes, so the output features are the UMMA M dimension
// (128 per CTA) and the activation rows the N dimension; D[m, n] lives in TMEM with one
// output feature per lane, so the epilogue writes consecutive features per warp.
// Warp 0 issues TMA loads into a 4-stage ring, warp 1 issues the UMMAs, all four warps
// run the epilogue. The absorb kernel also writes q_ext's rotary slots.
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

namespace {
constexpr int kWgStages = 4;
constexpr int kWgABytes = 128 * 128;  // 128 x 64 bf16 weight tile (two 64x64 boxes for W_UK)

template <int NR>
struct WgLayout {
  static constexpr int kB = NR * 128;                 // NR rows x 64 bf16
  static constexpr int kStage = kWgABytes + kB;
  static constexpr int kBars = kStage * kWgStages;
  static constexpr int kTotal = kBars + 256 + 1024;   // barriers + alignment slack
};

MLA_DEVICE uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
}  // namespace

template <int NR>
__global__ void __launch_bounds__(128, 1) wgemm_kernel(const __grid_constant__ WGemmParams p) {
  using Lay = WgLayout<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + Lay::kBars);
  uint64_t* empty = full + kWgStages;
  uint64_t* done = empty + kWgStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int n0 = blockIdx.z * NR;
  const int nk = (p.K + 63) / 64;
  constexpr uint32_t kCols = NR < 32 ? 32 : NR;
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWgStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      prefetch_tensormap(&p.tm_w);
      prefetch_tensormap(&p.tm_x);
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int st = kb % kWgStages;
        if (kb >= kWgStages && !mbar_wait(&empty[st], ((kb / kWgStages) - 1) & 1, wc)) break;
        uint8_t* a = base + st * Lay::kStage;
        uint8_t* b = a + kWgABytes;
        mbar_arrive_expect_tx(&full[st], Lay::kStage);
        if (p.a_mn) {
          tma_load_3d(a, &p.tm_w, m0, kb * 64, h, &full[st]);
          tma_load_3d(a + 8192, &p.tm_w, m0 + 64, kb * 64, h, &full[st]);
        } else {
          tma_load_3d(a, &p.tm_w, kb * 64, m0, h, &full[st]);
        }
        tma_load_3d(b, &p.tm_x, kb * 64, h, n0, &full[st]);
      }
      // never leave with copies in flight into this CTA's shared memory
      for (int j = (kb > kWgStages ? kb - kWgStages : 0); j < kb; ++j)
        mbar_wait_bounded(&full[j % kWgStages], (j / kWgStages) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = make_idesc_bf16(128, NR, p.a_mn, 0);
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % kWgStages;
        if (!mbar_wait(&full[st], (kb / kWgStages) & 1, wc)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(base + st * Lay::kStage);
        const uint32_t b = a + kWgABytes;
        const int rem = p.K - kb * 64;
        const int nkk = rem >= 64 ? 4 : (rem + 15) / 16;
        for (int kk = 0; kk < nkk; ++kk) {
          const uint64_t ad = p.a_mn ? make_sdesc(a + kk * 2048, 8192, 1024, kSw128)
                                     : make_sdesc(a + kk * 32, 16, 1024, kSw128);
          const uint64_t bd = make_sdesc(b + kk * 32, 16, 1024, kSw128);
          umma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0);
        }
        umma_commit(&empty[st]);
      }
      umma_commit(done);
    }
    __syncwarp();
  }

  // rotary slots of q_ext (absorb only), written by the first M tile of each head
  if (p.q_pe != nullptr && blockIdx.x == 0 && p.rope_dim > 0) {
    const int G = p.groups, dr = p.rope_dim, half = dr / 2;
    const int gh = h / (p.heads / G);
    const int nrows = min(NR, p.rows - n0);
    const int width = G * dr;
    for (int idx = threadIdx.x; idx < nrows * width; idx += 128) {
      const int n = n0 + idx / width;
      const int k = idx % width;
      const int g = k / dr;
      const int j = k % dr;
      float y = 0.0f;
      if (g == gh) {
        const int jj = j < half ? j : j - half;
        const uint16_t* q = p.q_pe + (int64_t(n) * p.heads + h) * dr;
        const float x0 = bf16_bits_to_f32(q[jj]);
        const float x1 = bf16_bits_to_f32(q[jj + half]);
        const int64_t ci = (int64_t(n) * G + g) * half + jj;
        const float c = p.rope_cos[ci];
        const float s = p.rope_sin[ci];
        y = j < half ? __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s))
                     : __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
      }
      p.out[int64_t(n) * p.out_row_stride + int64_t(h) * p.out_head_stride + p.M + k] =
          f32_to_bf16_rne(y);
    }
  }

  // epilogue: lane (32*warp + lane) holds output feature m for every row n of the tile
  const bool ok = mbar_wait(done, 0, wc);
  tc_fence_after();
  if (ok) {
    const int m = m0 + warp * 32 + lane;
    const float bias = (p.bias != nullptr && m < p.M)
                           ? bf16_bits_to_f32(p.bias[int64_t(h) * p.M + m]) : 0.0f;
    uint16_t* out = p.out + int64_t(h) * p.out_head_stride + m;
#pragma unroll
    for (int c0 = 0; c0 < NR; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + c0, v);
      tmem_wait_ld();
      if (m < p.M) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = n0 + c0 + j;
          if (n < p.rows) out[int64_t(n) * p.out_row_stride] = f32_to_bf16_rne(v[j] + bias);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

template <int NR>
static cudaError_t launch_wgemm_nr(const WGemmParams& p, cudaStream_t stream) {
  const int smem = WgLayout<NR>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(wgemm_kernel<NR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.M + 127) / 128, p.heads, (p.rows + NR - 1) / NR);
  wgemm_kernel<NR><<<grid, 128, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wgemm(const WGemmParams& p, int nr, cudaStream_t stream) {
  switch (nr) {
    case 16: return launch_wgemm_nr<16>(p, stream);
    case 32: return launch_wgemm_nr<32>(p, stream);
    case 64: return launch_wgemm_nr<64>(p, stream);
    case 128: return launch_wgemm_nr<128>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
