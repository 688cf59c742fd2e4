// decode.cu - mla_decode_attn on sm_100a: paged, split-KV absorbed attention over the
// latent cache, plus the log-sum-exp combine of the splits.
//
// Formulation. Every query row (i, h) of a sequence scores the SAME cache rows, so the
// CTA keeps the query block resident and streams the cache once:
//   S^T[tok, n] = C[tok, :] . Q[n, :]          UMMA M=64 tokens, N=NCOL rows, K = D
//   O^T[c, n]  += C[tok, c]^T P^T[tok, n]      UMMA M=128 latent, N=NCOL, K = 64 tokens
// with C a 64-token page of the cache (row = [c_kv | rotated keys]), Q = q_ext rows, and
// P^T the softmax weights written by the softmax warps. Putting tokens on M keeps N (the
// query rows, 4..64) free of padding and puts O^T's latent on TMEM lanes, so O^T needs
// only ceil(r/128) * NCOL TMEM columns. The same TMA-loaded, 128B-swizzled page is read
// K-major for S^T and MN-major for O^T.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 UMMA issuer + TMEM owner, warps 2-5
// softmax (one token per lane in lanes 0-15 of each TMEM sub-partition, as the M=64
// accumulator layout places rows 16*sp..16*sp+15 in lanes 32*sp..32*sp+15) and epilogue.
//
// Online softmax in the log2 domain with a lazily updated per-row reference max: the
// reference only moves when some score exceeds it by more than 8 (so unnormalised
// weights stay <= 256); then the new tile max is reduced across the CTA and O^T and the
// running sums are rescaled. Per-thread partial row sums are reduced once at the end.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mla {

namespace {

constexpr int kThreads = 192;
constexpr int kBlkBytes = kDecodeTok * 128;   // one 64 x 64 bf16 block, 8 KB
constexpr float kLazyThreshold = 8.0f;        // log2 units
constexpr float kLn2 = 0.69314718055994530942f;

struct DecodeLayout {
  uint32_t q_off, slot_off, pt_off, red_off, m_off, flag_off, misc_off, bar_off, total;
};

__host__ __device__ inline uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline DecodeLayout decode_layout(int ncol, int nblk, int slot_blocks,
                                                      int nslot, int npt) {
  DecodeLayout L;
  uint32_t off = 0;
  L.q_off = off;
  off += round_up(uint32_t(nblk) * ncol * 128, 1024);
  L.slot_off = off;
  off += uint32_t(nslot) * slot_blocks * kBlkBytes;
  L.pt_off = off;
  off += uint32_t(npt) * round_up(uint32_t(kDecodeTok) * ncol * 2, 1024);
  L.red_off = off;                 // float red[4][64]
  off += 4 * 64 * 4;
  L.m_off = off;                   // float m_ref[64]
  off += 64 * 4;
  L.flag_off = off;                // int flags[2][4]
  off += 2 * 4 * 4;
  L.misc_off = off;                // uint32 tmem base, int abort flag
  off += 16;
  L.bar_off = round_up(off, 8);    // mbarriers
  off = L.bar_off + 8 * (nslot * nblk + nslot + 1 + 2 * 4);
  L.total = off + 1024;            // slack for 1024-byte alignment of the base
  return L;
}

MLA_DEVICE uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int NCOL>
MLA_DEVICE void tmem_ld_cols(uint32_t taddr, float* v) {
#pragma unroll
  for (int c = 0; c < NCOL; c += 16) tmem_ld16(taddr + c, v + c);
}

template <int NCOL>
MLA_DEVICE void tmem_st_cols(uint32_t taddr, const float* v) {
#pragma unroll
  for (int c = 0; c < NCOL; c += 16) tmem_st16(taddr + c, v + c);
}

__host__ __device__ constexpr SmemSwizzle pt_swizzle(int ncol) {
  return ncol == 64 ? kSw128 : (ncol == 32 ? kSw64 : kSw32);
}

}  // namespace

size_t decode_smem_bytes(int ncol, int nblk, int slot_blocks, int nslot, int npt) {
  return decode_layout(ncol, nblk, slot_blocks, nslot, npt).total;
}

template <int NCOL>
__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const DecodeLayout lay = decode_layout(NCOL, p.nblk, p.slot_blocks, p.nslot, p.npt);
  uint8_t* q_smem = base + lay.q_off;
  uint8_t* slots = base + lay.slot_off;
  uint8_t* pt = base + lay.pt_off;
  float* red = reinterpret_cast<float*>(base + lay.red_off);
  float* m_ref = reinterpret_cast<float*>(base + lay.m_off);
  int* flags = reinterpret_cast<int*>(base + lay.flag_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + lay.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + lay.misc_off + 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + lay.bar_off);
  uint64_t* full = bars;                                        // [slot][blk]
  uint64_t* empty = full + p.nslot * p.nblk;                    // [slot]
  uint64_t* q_full = empty + kDecodeMaxSlots;
  uint64_t* s_full = q_full + 1;                                // [2]
  uint64_t* s_free = s_full + 2;                                // [2]
  uint64_t* p_full = s_free + 2;                                // [2]
  uint64_t* pv_done = p_full + 2;                               // [2]

  constexpr uint32_t kPtBytes = ((kDecodeTok * NCOL * 2) + 1023) / 1024 * 1024;
  constexpr uint32_t kQBlk = NCOL * 128;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int cg = blockIdx.y;
  const int b = blockIdx.z;
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nslot; ++s) {
      for (int k = 0; k < p.nblk; ++k) mbar_init(&full[s * p.nblk + k], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- work of this CTA: tiles [t0, t0 + ntl) of sequence b --------------------------
  int L = p.seq_lens[b];
  const bool len_ok = L >= p.q_len && L <= p.max_seq_len &&
                      int64_t(L) <= int64_t(p.max_pages) * kDecodeTok;
  if (!len_ok) {
    if (threadIdx.x == 0 && p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
    L = 0;
  }
  const int n_tiles = (L + kDecodeTok - 1) / kDecodeTok;
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(n_tiles, t0 + p.tiles_per_split);
  const int ntl = t1 > t0 ? t1 - t0 : 0;

  if (warp == 0) {
    // ===================================== TMA producer ==================================
    if (ntl > 0 && elect_one()) {
      prefetch_tensormap(&p.tm_cache);
      prefetch_tensormap(&p.tm_q);
      mbar_arrive_expect_tx(q_full, p.nblk * kQBlk);
      for (int k = 0; k < p.nblk; ++k)
        tma_load_3d(q_smem + k * kQBlk, &p.tm_q, k * 64, cg * NCOL, b, q_full);
      const int32_t* bt = p.block_table + int64_t(b) * p.max_pages;
      int jj = 0;
      for (; jj < ntl; ++jj) {
        const int slot = jj % p.nslot;
        if (jj >= p.nslot && !mbar_wait(&empty[slot], ((jj / p.nslot) - 1) & 1, wc)) break;
        int32_t page = bt[t0 + jj];
        if (page < 0 || page >= p.num_pages) {
          if (p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
          page = 0;
        }
        uint8_t* sbase = slots + slot * p.slot_blocks * kBlkBytes;
        for (int k = 0; k < p.nblk; ++k) {
          uint64_t* fb = &full[slot * p.nblk + k];
          mbar_arrive_expect_tx(fb, kBlkBytes);
          tma_load_2d(sbase + k * kBlkBytes, &p.tm_cache, k * 64, page * kDecodeTok, fb);
        }
      }
      // Drain: never leave while copies into this CTA's shared memory are in flight.
      mbar_wait_bounded(q_full, 0, 200000000ull);
      for (int j = (jj > p.nslot ? jj - p.nslot : 0); j < jj; ++j)
        for (int k = 0; k < p.nblk; ++k)
          mbar_wait_bounded(&full[(j % p.nslot) * p.nblk + k], (j / p.nslot) & 1,
                            200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ===================================== UMMA issuer ===================================
    if (ntl > 0 && elect_one()) {
      const uint32_t idesc_s = make_idesc_bf16(64, NCOL, 0, 0);
      const uint32_t idesc_o = make_idesc_bf16(128, NCOL, 1, 1);
      const uint32_t q_addr = smem_u32(q_smem);
      const uint32_t slot_addr0 = smem_u32(slots);
      const uint32_t pt_addr0 = smem_u32(pt);
      const uint32_t pt_sbo = 8 * NCOL * 2;
      const SmemSwizzle pt_sw = pt_swizzle(NCOL);
      bool ok = mbar_wait(q_full, 0, wc);

      auto issue_pv = [&](int t) -> bool {
        const int pb = t & 1;
        const int slot = t % p.nslot;
        if (!mbar_wait(&p_full[pb], (t >> 1) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t sa = slot_addr0 + slot * p.slot_blocks * kBlkBytes;
        const uint32_t pa = pt_addr0 + (t % p.npt) * kPtBytes;
        for (int c = 0; c < p.nch; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc(sa + 2 * c * kBlkBytes + kk * 2048, kBlkBytes, 1024, kSw128);
            const uint64_t bd = make_sdesc(pa + kk * 16 * NCOL * 2, kPtBytes, pt_sbo, pt_sw);
            umma_bf16(tmem + (2 + c) * NCOL, ad, bd, idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&pv_done[pb]);
        umma_commit(&empty[slot]);
        return true;
      };

      for (int jj = 0; ok && jj < ntl; ++jj) {
        const int slot = jj % p.nslot;
        const int sb = jj & 1;
        if (jj >= 2 && !mbar_wait(&s_free[sb], ((jj - 2) >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = slot_addr0 + slot * p.slot_blocks * kBlkBytes;
        for (int k = 0; k < p.nblk; ++k) {
          if (!mbar_wait(&full[slot * p.nblk + k], (jj / p.nslot) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const int rem = p.D - k * 64;
          const int nkk = rem >= 64 ? 4 : (rem + 15) / 16;
          for (int kk = 0; kk < nkk; ++kk) {
            const uint64_t ad = make_sdesc(sa + k * kBlkBytes + kk * 32, 16, 1024, kSw128);
            const uint64_t bd = make_sdesc(q_addr + k * kQBlk + kk * 32, 16, 1024, kSw128);
            umma_bf16(tmem + sb * NCOL, ad, bd, idesc_s, (k | kk) != 0 ? 1u : 0u);
          }
        }
        if (!ok) break;
        umma_commit(&s_full[sb]);
        if (jj >= 1 && !issue_pv(jj - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(ntl - 1);
    }
    __syncwarp();
  } else {
    // ================================ softmax + epilogue =================================
    const int sp = warp & 3;                  // TMEM sub-partition this warp may access
    const int wi = warp - 2;                  // index among the 4 softmax warps
    const uint32_t lane_base = uint32_t(sp * 32) << 16;
    const bool has_tok = lane < 16;
    const int tok = 16 * sp + lane;           // token of this lane inside the tile
    const int qH = p.qH;
    const int last_pos = L - p.q_len;         // position of query row 0
    float l_part[NCOL];
#pragma unroll
    for (int n = 0; n < NCOL; ++n) l_part[n] = 0.0f;
    if (threadIdx.x - 64 < NCOL) m_ref[threadIdx.x - 64] = -INFINITY;
    named_bar_sync(1, 128);

    for (int jj = 0; jj < ntl; ++jj) {
      const int sb = jj & 1;
      const int tile = t0 + jj;
      // warp-uniform: the TMEM load below is a warp-collective instruction
      const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (jj >> 1) & 1, wc));
      float s[NCOL];
      if (got) {
        tc_fence_after();
        tmem_ld_cols<NCOL>(tmem + lane_base + sb * NCOL, s);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&s_free[sb]);

      const int pos = tile * kDecodeTok + tok;
      const bool tok_ok = got && has_tok && pos < L;
      bool exceed = false;
#pragma unroll
      for (int n = 0; n < NCOL; ++n) {
        const int f = cg * NCOL + n;
        const int qi = f / p.num_heads;
        const bool vis = tok_ok && f < qH && (!p.causal || pos <= last_pos + qi);
        s[n] = vis ? s[n] * p.scale_log2 : -INFINITY;
        exceed |= s[n] > m_ref[n] + kLazyThreshold;
      }
      exceed = __any_sync(0xffffffffu, exceed);
      if (lane == 0) flags[(jj & 1) * 4 + wi] = exceed ? 1 : 0;
      named_bar_sync(1, 128);
      const bool upd = (flags[(jj & 1) * 4 + 0] | flags[(jj & 1) * 4 + 1] |
                        flags[(jj & 1) * 4 + 2] | flags[(jj & 1) * 4 + 3]) != 0;
      if (upd) {
        // tile max per query row across the 64 tokens (16 lanes x 4 warps)
        float tmax[NCOL];
#pragma unroll
        for (int n = 0; n < NCOL; ++n) {
          float v = s[n];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          tmax[n] = v;
        }
        if (lane == 0) {
#pragma unroll
          for (int n = 0; n < NCOL; ++n) red[wi * 64 + n] = tmax[n];
        }
        named_bar_sync(1, 128);
        float alpha[NCOL];
        bool rescale = false;
#pragma unroll
        for (int n = 0; n < NCOL; ++n) {
          const float mo = m_ref[n];
          const float mn = fmaxf(fmaxf(mo, red[n]),
                                 fmaxf(fmaxf(red[64 + n], red[128 + n]), red[192 + n]));
          alpha[n] = (mo == -INFINITY) ? 0.0f : ex2_approx(mo - mn);
          rescale |= (mo != -INFINITY) && (mn != mo);
          tmax[n] = mn;
          l_part[n] *= alpha[n];
        }
        if (rescale && jj > 0) {
          // O^T holds tiles < jj: wait for the last of them, then scale its columns
          if (__all_sync(0xffffffffu, mbar_wait(&pv_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, wc))) {
            tc_fence_after();
            for (int c = 0; c < p.nch; ++c) {
              float o[NCOL];
              const uint32_t ta = tmem + lane_base + (2 + c) * NCOL;
              tmem_ld_cols<NCOL>(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int n = 0; n < NCOL; ++n) o[n] *= alpha[n];
              tmem_st_cols<NCOL>(ta, o);
            }
            tmem_wait_st();
          }
        }
        named_bar_sync(1, 128);
        if (threadIdx.x - 64 < NCOL) {
          float v = -INFINITY;
#pragma unroll
          for (int n = 0; n < NCOL; ++n) v = (n == int(threadIdx.x) - 64) ? tmax[n] : v;
          m_ref[threadIdx.x - 64] = v;
        }
        named_bar_sync(1, 128);
      }

      // unnormalised weights p = 2^(s - m_ref), bf16, into the P^T buffer of this tile;
      // the buffer is free once the PV product that last read it has completed
      if (jj >= p.npt) mbar_wait(&pv_done[(jj - p.npt) & 1], ((jj - p.npt) >> 1) & 1, wc);
      uint32_t packed[NCOL / 2];
#pragma unroll
      for (int n = 0; n < NCOL; n += 2) {
        const float p0 = s[n] == -INFINITY ? 0.0f : ex2_approx(s[n] - m_ref[n]);
        const float p1 = s[n + 1] == -INFINITY ? 0.0f : ex2_approx(s[n + 1] - m_ref[n + 1]);
        l_part[n] += p0;
        l_part[n + 1] += p1;
        packed[n / 2] = cvt_bf16x2(p0, p1);
      }
      if (has_tok) {
        uint8_t* row = pt + (jj % p.npt) * kPtBytes;
        constexpr uint32_t kRowBytes = NCOL * 2;
        constexpr uint32_t kChunkMask = kRowBytes / 16 - 1;
#pragma unroll
        for (int ch = 0; ch < NCOL / 8; ++ch) {
          const uint32_t off = tok * kRowBytes + ch * 16;
          const uint32_t phys = off ^ (((off >> 7) & kChunkMask) << 4);
          *reinterpret_cast<uint4*>(row + phys) =
              make_uint4(packed[ch * 4 + 0], packed[ch * 4 + 1], packed[ch * 4 + 2], packed[ch * 4 + 3]);
        }
        // cache rows past the context may hold anything (even NaN): zero them so that
        // 0-weight x garbage cannot reach O^T
        if (tile == n_tiles - 1 && pos >= L) {
          uint8_t* sbase = slots + (jj % p.nslot) * p.slot_blocks * kBlkBytes;
          for (int k = 0; k < 2 * p.nch; ++k) {
            uint4* rowp = reinterpret_cast<uint4*>(sbase + k * kBlkBytes + tok * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) rowp[ch] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }

    // ---------------------------------- epilogue ------------------------------------------
    bool fin = true;
    if (ntl > 0) {
      fin = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ntl - 1) & 1], ((ntl - 1) >> 1) & 1, wc));
      tc_fence_after();
    }
#pragma unroll
    for (int n = 0; n < NCOL; ++n) {
      float v = l_part[n];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      l_part[n] = v;
    }
    if (lane == 0) {
#pragma unroll
      for (int n = 0; n < NCOL; ++n) red[wi * 64 + n] = l_part[n];
    }
    named_bar_sync(1, 128);
    float inv_l[NCOL];
#pragma unroll
    for (int n = 0; n < NCOL; ++n) {
      const float l = red[n] + red[64 + n] + red[128 + n] + red[192 + n];
      inv_l[n] = l > 0.0f ? 1.0f / l : 0.0f;
    }
    const bool aborted = __any_sync(0xffffffffu, !fin || *abort_flag != 0);
    const int cols_here = min(NCOL, qH - cg * NCOL);
    const int64_t part_base = (int64_t(b) * p.col_groups + cg) * p.splits + split;
    // lse (natural log) of each query row
    const int tid = threadIdx.x - 64;
    if (tid < cols_here) {
      const float l = red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
      const float v = (l > 0.0f && !aborted) ? (m_ref[tid] + __log2f(l)) * kLn2 : -INFINITY;
      if (p.splits == 1) p.lse[int64_t(b) * qH + cg * NCOL + tid] = v;
      else p.part_lse[part_base * NCOL + tid] = v;
    }
    // O^T: this thread owns latent row 128*c + 32*sp + lane of every chunk c
    for (int c = 0; c < p.nch; ++c) {
      float o[NCOL];
      if (ntl > 0 && !aborted) {
        tmem_ld_cols<NCOL>(tmem + lane_base + (2 + c) * NCOL, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int n = 0; n < NCOL; ++n) o[n] = 0.0f;
      }
      const int lat = 128 * c + 32 * sp + lane;
      if (lat < p.r) {
        if (p.splits == 1) {
          uint16_t* dst = p.o_latent + (int64_t(b) * qH + cg * NCOL) * p.r + lat;
#pragma unroll
          for (int n = 0; n < NCOL; ++n)
            if (n < cols_here) dst[int64_t(n) * p.r] = f32_to_bf16_rne(o[n] * inv_l[n]);
        } else {
          float* dst = p.part_o + part_base * NCOL * p.r + lat;
#pragma unroll
          for (int n = 0; n < NCOL; ++n)
            if (n < cols_here) dst[int64_t(n) * p.r] = o[n] * inv_l[n];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

// ---- split merge: lse = log sum_s e^{lse_s}, o = sum_s e^{lse_s - lse} o_s ---------------
__global__ void __launch_bounds__(128) mla_combine_kernel(CombineParams p) {
  const int f = blockIdx.x;   // query row (i, h) of sequence b
  const int b = blockIdx.y;
  const int cg = f / p.ncol;
  const int n = f % p.ncol;
  const int64_t base = (int64_t(b) * p.col_groups + cg) * p.splits;
  float mx = -INFINITY;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.part_lse[(base + s) * p.ncol + n]);
  float wsum = 0.0f;
  for (int s = 0; s < p.splits; ++s) {
    const float ls = p.part_lse[(base + s) * p.ncol + n];
    wsum += ls == -INFINITY ? 0.0f : expf(ls - mx);
  }
  const float lse = mx == -INFINITY ? -INFINITY : mx + logf(wsum);
  if (threadIdx.x == 0) p.lse[int64_t(b) * p.qH + f] = lse;
  for (int c = threadIdx.x; c < p.r; c += blockDim.x) {
    float acc = 0.0f;
    for (int s = 0; s < p.splits; ++s) {
      const float ls = p.part_lse[(base + s) * p.ncol + n];
      if (ls == -INFINITY) continue;
      acc += expf(ls - lse) * p.part_o[((base + s) * p.ncol + n) * p.r + c];
    }
    p.o_latent[(int64_t(b) * p.qH + f) * p.r + c] = f32_to_bf16_rne(acc);
  }
}

template <int NCOL>
static cudaError_t launch_decode_n(const DecodeParams& p, dim3 grid, size_t smem,
                                   cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<NCOL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  mla_decode_kernel<NCOL><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, int ncol, dim3 grid, size_t smem,
                          cudaStream_t stream) {
  switch (ncol) {
    case 16: return launch_decode_n<16>(p, grid, smem, stream);
    case 32: return launch_decode_n<32>(p, grid, smem, stream);
    case 64: return launch_decode_n<64>(p, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  dim3 grid(p.qH, p.batch);
  mla_combine_kernel<<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
