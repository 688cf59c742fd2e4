// decode.cu - mla_decode_attn on sm_100a for blocks of up to 64 query rows: paged,
// split-KV absorbed attention over the latent cache (the merge of split pieces is in
// combine.cu).
//
// Formulation. Every query row (i, h) of a sequence scores the SAME cache rows, so the
// CTA keeps a block of NCOL query rows resident and streams the cache pages once:
//   S^T[tok, n] = C[tok, :] . Q[n, :]          UMMA M=64 tokens, N=NCOL rows, K = D
//   O^T[c, n]  += C[tok, c]^T P^T[tok, n]      UMMA M=128 latent, N=NCOL, K = 64 tokens
// with C one 64-token page of the cache (row = [c_kv | rotated keys]), Q the q_ext rows
// and P^T the softmax weights written by the softmax warps. Tokens on M keep N (4..64
// query rows) free of padding and put O^T's latent on TMEM lanes, so O^T needs only
// ceil(r/128) * NCOL TMEM columns. The same TMA-loaded, 128B-swizzled page is read
// K-major for S^T and MN-major for O^T.
//
// Schedule. A "unit" is (sequence b, block cg of NCOL query rows); its work is
// ceil(L_b / 64) page tiles. The units' tiles are laid end to end and cut into gridDim.x
// equal ranges, one per CTA, so ragged lengths balance. A CTA walks the units its range
// touches; a unit it holds whole is written straight to o_latent / lse, a unit cut
// between CTAs leaves one normalised partial per piece (o in bf16, lse in fp32), merged
// afterwards by the merge kernels of combine.cu with the log-sum-exp identity.
//
// Roles (224 threads): warp 0 TMA producer, warp 1 S^T issuer and TMEM owner, warps 2-5
// softmax and epilogue, warp 6 PV issuer. (Issued by one lane of a softmax warp, the 16
// PV products of a page took ~2.5x their issue cost; a warp of their own issues them at
// the rate the tensor core accepts them.) In the M=64 accumulator layout rows 16*sp..16*sp+15 sit in lanes
// 32*sp..32*sp+15 of TMEM sub-partition sp; the 16x32bx2 load gives each of those 16
// tokens to two threads, one per half of the NCOL columns.
//
// Online softmax in the log2 domain with a lazily moved reference max per query row:
// it moves only when a score exceeds it by more than 8 (unnormalised weights stay <= 256);
// then the tile max is reduced over the CTA and O^T and the running sums are rescaled.
#include <math.h>

#include <algorithm>

#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

// Optional per-tile timeline of CTA 0 (compile with -DMLA_TRACE; read with mla_trace_read).
// Events: 0 producer starts a tile, 1 S issued (all blocks landed), 2 S committed, 3 PV
// committed, 4 softmax sees S, 5 after the vote barrier, 6 P buffer free, 7 P written
// and PV about to be issued, 8 producer finished issuing the tile, 9 the whole page landed.
#ifdef MLA_TRACE
constexpr int kTraceTiles = 512;
__device__ unsigned long long g_mla_trace[10 * kTraceTiles + 1];
#define MLA_TRACE_AT(ev, idx)                                                         \
  do {                                                                                \
    if (blockIdx.x == 0 && (idx) < kTraceTiles) g_mla_trace[(ev) * kTraceTiles + (idx)] = clock64(); \
  } while (0)
#else
#define MLA_TRACE_AT(ev, idx) \
  do {                       \
  } while (0)
#endif

namespace {

constexpr int kThreads = 224;
constexpr int kBlkBytes = kDecodeTok * 128;   // one 64 x 64 bf16 block, 8 KB
constexpr float kLazyThreshold = 8.0f;        // log2 units
// Initial reference max: finite, so a masked score (-inf) minus it is exactly -inf (weight
// 0) and any finite score exceeds it, forcing the first real reference to be computed.
constexpr float kRefInit = -3.0e38f;
constexpr float kLn2 = 0.69314718055994530942f;
// misc ints: [0,8) vote flags, 8 TMEM base, 9 abort flag, [10,16) schedule, [16,22) warp
// sums, [23,25) reference-moved flags; 32 reserved.
constexpr int kMiscInts = 32;

struct DecodeLayout {
  uint32_t q_off, slot_off, pt_off, red_off, alpha_off, mref_off, misc_off, bar_off, total;
};

__host__ __device__ inline uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ constexpr int num_bars(int nslot) { return 2 * nslot + 10; }

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
  L.red_off = off;                 // float red[4][64]: per-warp column partials
  off += 4 * 64 * 4;
  L.alpha_off = off;               // float alpha[64]: O^T rescale factor per column
  off += 64 * 4;
  L.mref_off = off;                // float mref[64]: reference max per column
  off += 64 * 4;
  L.misc_off = off;                // int misc[kMiscInts], index map in the kernel
  off += 4 * kMiscInts;
  L.bar_off = round_up(off, 8);
  off = L.bar_off + 8 * num_bars(nslot);
  L.total = off + 1024;            // slack for 1024-byte alignment of the base
  return L;
}

MLA_DEVICE uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 16x32bx2 TMEM load of the M=64 S^T accumulator: threads 0-15 read lanes 0-15 of the
// warp's sub-partition at columns [c, c+HALF), threads 16-31 the same lanes at
// [c+HALF, c+2*HALF).
template <int HALF>
MLA_DEVICE void tmem_ld_s(uint32_t taddr, float* v);

template <>
MLA_DEVICE void tmem_ld_s<8>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], 8;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

template <>
MLA_DEVICE void tmem_ld_s<16>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <>
MLA_DEVICE void tmem_ld_s<32>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
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
  constexpr int HALF = NCOL / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  const DecodeLayout lay = decode_layout(NCOL, p.nblk, p.slot_blocks, p.nslot, p.npt);
  uint8_t* q_smem = base + lay.q_off;
  uint8_t* slots = base + lay.slot_off;
  uint8_t* pt = base + lay.pt_off;
  float* red = reinterpret_cast<float*>(base + lay.red_off);
  float* alpha_s = reinterpret_cast<float*>(base + lay.alpha_off);
  float* mref_s = reinterpret_cast<float*>(base + lay.mref_off);
  int* misc = reinterpret_cast<int*>(base + lay.misc_off);
  int* flags = misc;                                   // [2][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 8);
  volatile int* abort_flag = misc + 9;
  int* sched = misc + 10;                              // b_a, s_a, r0, r1, per, scan carry
  int* warp_sum = misc + 16;                           // [6]
  int* chg_flag = misc + 23;                           // [2] reference moved, per half
  static_assert(23 + 2 <= kMiscInts, "misc ints overflow into the mbarriers");
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + lay.bar_off);
  // One TMA barrier per slot for all boxes of a page: S^T starts once the whole page has
  // landed. Every mbarrier operation on the S^T issuer's path costs a few hundred cycles, and
  // one barrier per page measured faster than one per 64-column box.
  uint64_t* full = bars;                               // [slot]
  uint64_t* empty = full + p.nslot;                    // [slot]
  uint64_t* q_full = empty + p.nslot;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_empty + 1;                      // [2]
  uint64_t* s_free = s_full + 2;                       // [2]
  uint64_t* pv_done = s_free + 2;                      // [2]
  uint64_t* p_full = pv_done + 2;                      // [npt] P^T written (4 softmax warps)

  constexpr uint32_t kPtBytes = ((kDecodeTok * NCOL * 2) + 1023) / 1024 * 1024;
  constexpr uint32_t kQBlk = NCOL * 128;
  const uint32_t slot_bytes = uint32_t(p.slot_blocks) * kBlkBytes;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cg = int(blockIdx.x) % p.col_groups;       // row block of this CTA
  const int vc = int(blockIdx.x) / p.col_groups;       // index among the CTAs of that block
  const int vgrid = int(gridDim.x) / p.col_groups;
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nslot; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&p_full[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }

  // set-up above may overlap the previous kernel; from here on global memory is touched
  grid_dep_wait();
  grid_dep_launch();
  // ---- schedule: this CTA's tile range [r0, r1) in its row block, first sequence -------
  // The row blocks of a sequence are worked on in lockstep by neighbouring CTAs, so the
  // second read of every page is served from L2.
  find_tile_range<kThreads>(p, vc, vgrid, blockIdx.x == 0, warp_sum, sched);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int r0 = sched[2], r1 = sched[3], per = sched[4];
  const bool has_work = sched[0] >= 0 && r0 < r1;

  if (warp == 0) {
    // ===================================== TMA producer ==================================
    if (has_work && elect_one()) {
      prefetch_tensormap(&p.tm_cache);
      prefetch_tensormap(&p.tm_q);
      if (blockIdx.x == 0) *p.range_len = per;
      UnitWalk w{sched[0], sched[1]};
      int jj = 0, pc = 0;
      SlotRing ring(p.nslot);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b, ++pc) {
        w.load(p, cg);
        p.unit_start[w.u] = w.s;   // same value from every CTA that touches the unit
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        if (pc > 0 && !mbar_wait(q_empty, (pc - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, p.nblk * kQBlk);
        for (int k = 0; k < p.nblk; ++k)
          tma_load_3d(q_smem + k * kQBlk, &p.tm_q, k * 64, cg * NCOL, w.b, q_full);
        const int32_t* bt = p.block_table + int64_t(w.b) * p.max_pages;
        for (int t = tb; t < te; ++t, ++jj, ring.next()) {
          const int slot = ring.slot;
          // the page id is read before the wait, so its round trip overlaps it
          int32_t page = bt[t - w.s];
          if (jj >= p.nslot && !mbar_wait(&empty[slot], (ring.round - 1) & 1, wc)) {
            ok = false;
            break;
          }
          MLA_TRACE_AT(0, jj);
          if (page < 0 || page >= p.num_pages) {
            if (p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
            page = 0;
          }
          uint8_t* sbase = slots + slot * slot_bytes;
          uint64_t* fb = &full[slot];
          mbar_arrive_expect_tx(fb, uint32_t(p.nblk) * kBlkBytes);
          for (int k = 0; k < p.nblk; ++k)
            tma_load_2d(sbase + k * kBlkBytes, &p.tm_cache, k * 64, page * kDecodeTok, fb);
          MLA_TRACE_AT(8, jj);
        }
      }
      // Drain: never leave while copies into this CTA's shared memory are in flight.
      if (pc > 0) mbar_wait_bounded(q_full, (pc - 1) & 1, 200000000ull);
      for (int j = (jj > p.nslot ? jj - p.nslot : 0); j < jj; ++j)
        mbar_wait_bounded(&full[j % p.nslot], (j / p.nslot) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ UMMA issuer for S^T ================================
    // S^T(j) is issued once the whole page has landed. The PV products are issued by the
    // softmax warps themselves, the moment P(j) is written.
    if (has_work && elect_one()) {
      const uint32_t idesc_s = make_idesc_bf16(64, NCOL, 0, 0);
      const uint64_t a0 = make_sdesc(smem_u32(slots), 16, 1024, kSw128);
      const uint64_t b0 = make_sdesc(smem_u32(q_smem), 16, 1024, kSw128);
      const int nk16 = (p.D + 15) / 16;              // K steps over the row width
      UnitWalk w{sched[0], sched[1]};
      int jj = 0, pc = 0;
      SlotRing ring(p.nslot);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b, ++pc) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        if (!mbar_wait(q_full, pc & 1, wc)) { ok = false; break; }
        for (int t = tb; ok && t < te; ++t, ++jj, ring.next()) {
          const int slot = ring.slot;
          const int sb = jj & 1;
          if (jj >= 2 && !mbar_wait(&s_free[sb], ((jj - 2) >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t soff = slot * slot_bytes;
          if (!mbar_wait(&full[slot], ring.round & 1, wc)) { ok = false; break; }
          tc_fence_after();
          MLA_TRACE_AT(9, jj);
          // K steps of 16 columns over the row width; the descriptors step 32 bytes within
          // a 64-column block and to the next block's start after its fourth step
          {
            const uint32_t dS = tmem + sb * NCOL;
            uint64_t ad = a0 + (soff >> 4), bd = b0;
            umma_bf16(dS, ad, bd, idesc_s, 0u);
            for (int i = 1; i < nk16; ++i) {
              const bool next_blk = (i & 3) == 0;
              ad += next_blk ? uint64_t((kBlkBytes - 96) >> 4) : uint64_t(2);
              bd += next_blk ? uint64_t((kQBlk - 96) >> 4) : uint64_t(2);
              umma_bf16(dS, ad, bd, idesc_s, 1u);
            }
          }
          MLA_TRACE_AT(1, jj);
          umma_commit(&s_full[sb]);
          MLA_TRACE_AT(2, jj);
          if (t == te - 1) umma_commit(q_empty);   // this piece's Q is no longer read
        }
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // =============================== UMMA issuer for PV ==================================
    // O^T += C^T P^T for page j once the four softmax warps have written P^T(j) and zeroed
    // the page's rows past the context; the first page of a piece overwrites O^T (the
    // softmax warps read the previous piece's O^T before they arrive on P^T's barrier).
    if (has_work && elect_one()) {
      const uint32_t idesc_o = make_idesc_bf16(128, NCOL, 1, 1);
      const uint64_t pa0 = make_sdesc(smem_u32(slots), kBlkBytes, 1024, kSw128);
      const uint64_t pb0 = make_sdesc(smem_u32(pt), kPtBytes, 8 * NCOL * 2, pt_swizzle(NCOL));
      UnitWalk w{sched[0], sched[1]};
      int jj = 0;
      SlotRing ring(p.nslot), pring(p.npt);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        for (int t = tb; t < te; ++t, ++jj, ring.next(), pring.next()) {
          if (!mbar_wait(&p_full[pring.slot], pring.round & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          MLA_TRACE_AT(7, jj);
          const bool first = (t == tb);
          // K-step outer, latent chunk inner: consecutive MMAs feed different accumulators;
          // descriptors stepped (16 tokens = 2 KB of C^T, 16 rows of P^T; 128 latent = 2
          // blocks)
          const uint64_t ad0 = pa0 + ((ring.slot * slot_bytes) >> 4);
          uint64_t bd = pb0 + ((pring.slot * kPtBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint64_t ad = ad0 + uint64_t(kk * (2048 >> 4));
            const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
            for (int c = 0; c < p.nch; ++c) {
              umma_bf16(tmem + (2 + c) * NCOL, ad, bd, idesc_o, acc);
              ad += uint64_t((2 * kBlkBytes) >> 4);
            }
            bd += uint64_t((16 * NCOL * 2) >> 4);
          }
          umma_commit(&pv_done[jj & 1]);
          umma_commit(&empty[ring.slot]);
          MLA_TRACE_AT(3, jj);
        }
      }
    }
    __syncwarp();
  } else if (has_work) {   // warps 2-5
    // ================================ softmax, epilogue ==================================
    const int sp = warp & 3;                  // TMEM sub-partition this warp may access
    const int wi = warp - 2;                  // index among the 4 softmax warps
    const int tid = threadIdx.x - 64;         // 0..127
    const uint32_t lane_base = uint32_t(sp * 32) << 16;
    const int tok = 16 * sp + (lane & 15);    // token of this thread inside the tile
    const int hf = lane >> 4;                 // which half of the columns
    const int c0 = hf * HALF;                 // first column of this thread
    const bool col_owner = (lane & 15) == 0;  // publishes its half-warp's column values
    const float c_log2 = p.scale_log2;

    UnitWalk w{sched[0], sched[1]};
    int jj = 0;
    SlotRing ring(p.nslot), pring(p.npt);
    for (; w.s < r1; w.s += w.tiles, ++w.b) {
      w.load(p, cg);
      const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
      const int L = w.L;
      const int last_full = p.causal ? L - p.q_len : L - 1;  // last position every row sees
      float m[HALF], l[HALF];
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        m[j] = kRefInit;
        l[j] = 0.0f;
      }
      for (int t = tb; t < te; ++t, ++jj, ring.next(), pring.next()) {
        const int sb = jj & 1;
        const uint32_t s_addr = tmem + lane_base + sb * NCOL;
        const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (jj >> 1) & 1, wc));
        if (threadIdx.x == 64) MLA_TRACE_AT(4, jj);
        const int tile_pos0 = (t - w.s) * kDecodeTok;
        const int pos = tile_pos0 + tok;
        const bool ragged = !got || tile_pos0 + kDecodeTok - 1 > last_full;
        // tt = s * c - m: the scaled score against the current reference (in place)
        float tt[HALF];
        if (got) {
          tc_fence_after();
          tmem_ld_s<HALF>(s_addr, tt);
          tmem_wait_ld();
        }
        if (ragged) {
          // row (i, h) sees token pos iff pos < L and (causal) pos <= L - q + i
#pragma unroll
          for (int j = 0; j < HALF; ++j) {
            const int qi = (cg * NCOL + c0 + j) / p.num_heads;
            const bool vis = got && pos < L && (!p.causal || pos <= L - p.q_len + qi);
            tt[j] = vis ? tt[j] : -INFINITY;
          }
        }
        float tmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < HALF; ++j) {
          tt[j] = fmaf(tt[j], c_log2, -m[j]);
          tmax = fmaxf(tmax, tt[j]);
        }
        const bool exceed = __any_sync(0xffffffffu, tmax > kLazyThreshold);
        if (lane == 0) flags[(jj & 1) * 4 + wi] = exceed ? 1 : 0;
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) MLA_TRACE_AT(5, jj);
        const int* fl = flags + (jj & 1) * 4;
        if ((fl[0] | fl[1] | fl[2] | fl[3]) != 0) {
          // Move the reference to the running column max of the scaled scores; the raw
          // scores are read again from TMEM (the S buffer is released only below).
          float s[HALF];
          if (got) {
            tmem_ld_s<HALF>(s_addr, s);
            tmem_wait_ld();
          }
#pragma unroll
          for (int j = 0; j < HALF; ++j) {
            if (ragged) {
              const int qi = (cg * NCOL + c0 + j) / p.num_heads;
              const bool vis = got && pos < L && (!p.causal || pos <= L - p.q_len + qi);
              s[j] = vis ? s[j] : -INFINITY;
            }
            float v = s[j] * c_log2;   // -inf stays -inf
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
            if (col_owner) red[wi * 64 + c0 + j] = v;
          }
          named_bar_sync(1, 128);
          bool chg = false;
#pragma unroll
          for (int j = 0; j < HALF; ++j) {
            const int n = c0 + j;
            const float tm = fmaxf(fmaxf(red[n], red[64 + n]), fmaxf(red[128 + n], red[192 + n]));
            const float mn = fmaxf(m[j], tm);
            const float a = ex2_approx(m[j] - mn);   // 0 while m is still kRefInit
            l[j] *= a;
            m[j] = mn;
            tt[j] = fmaf(s[j], c_log2, -mn);
            chg |= a != 1.0f;
            if (col_owner && wi == 0) alpha_s[n] = a;
          }
          if (col_owner && wi == 0) chg_flag[hf] = chg ? 1 : 0;
          named_bar_sync(1, 128);
          if (t > tb && (chg_flag[0] | chg_flag[1]) != 0) {
            // O^T already holds this piece's earlier tiles: scale every column of the
            // latent rows this thread owns (all threads see the same factors)
            const bool okw = __all_sync(0xffffffffu,
                                        mbar_wait(&pv_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, wc));
            if (okw) {
              tc_fence_after();
#pragma unroll 1
              for (int n0 = 0; n0 < NCOL; n0 += 16) {
                float a16[16];
#pragma unroll
                for (int n = 0; n < 16; ++n) a16[n] = alpha_s[n0 + n];
                for (int c = 0; c < p.nch; ++c) {
                  const uint32_t ta = tmem + lane_base + (2 + c) * NCOL + n0;
                  float o[16];
                  tmem_ld16(ta, o);
                  tmem_wait_ld();
#pragma unroll
                  for (int n = 0; n < 16; ++n) o[n] *= a16[n];
                  tmem_st16(ta, o);
                }
              }
              tmem_wait_st();
            }
          }
        }

        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);   // S buffer may be overwritten now

        // unnormalised weights p = 2^(s*c - m) into this tile's P^T buffer (bf16)
        if (jj >= p.npt) mbar_wait(&pv_done[(jj - p.npt) & 1], ((jj - p.npt) >> 1) & 1, wc);
        if (threadIdx.x == 64) MLA_TRACE_AT(6, jj);
        uint32_t packed[HALF / 2];
#pragma unroll
        for (int j = 0; j < HALF; j += 2) {
          const float p0 = ex2_approx(tt[j]);
          const float p1 = ex2_approx(tt[j + 1]);
          l[j] += p0;
          l[j + 1] += p1;
          packed[j / 2] = cvt_bf16x2(p0, p1);
        }
        const int slot = ring.slot;
        const int pbuf = pring.slot;
        {
          uint8_t* buf = pt + pbuf * kPtBytes;
          constexpr uint32_t kRowBytes = NCOL * 2;
          constexpr uint32_t kChunkMask = kRowBytes / 16 - 1;
#pragma unroll
          for (int ch = 0; ch < HALF / 8; ++ch) {
            const uint32_t off = tok * kRowBytes + (hf * (HALF / 8) + ch) * 16;
            const uint32_t phys = off ^ (((off >> 7) & kChunkMask) << 4);
            *reinterpret_cast<uint4*>(buf + phys) = make_uint4(
                packed[ch * 4 + 0], packed[ch * 4 + 1], packed[ch * 4 + 2], packed[ch * 4 + 3]);
          }
        }
        // cache rows past the context may hold anything (even NaN): zero them so that
        // 0-weight x garbage cannot reach O^T
        if (pos >= L) {
          uint8_t* sbase = slots + slot * slot_bytes;
          for (int k = hf; k < 2 * p.nch; k += 2) {
            uint4* rowp = reinterpret_cast<uint4*>(sbase + k * kBlkBytes + tok * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) rowp[ch] = make_uint4(0, 0, 0, 0);
          }
        }
        // P^T(j) and the zeroed rows are complete: hand the page to the PV issuer
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pbuf]);
      }

      // ---------------------------- epilogue of this piece --------------------------------
      const bool fin = __all_sync(0xffffffffu,
                                  mbar_wait(&pv_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, wc));
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        float v = l[j];
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        l[j] = v;
      }
      named_bar_sync(1, 128);   // every earlier reader of red / mref_s is done
      if (col_owner) {
#pragma unroll
        for (int j = 0; j < HALF; ++j) red[wi * 64 + c0 + j] = l[j];
      }
      if (col_owner && wi == 0) {
#pragma unroll
        for (int j = 0; j < HALF; ++j) mref_s[c0 + j] = m[j];
      }
      named_bar_sync(1, 128);
      const bool aborted = __any_sync(0xffffffffu, !fin || *abort_flag != 0);
      const bool whole = (tb == w.s) && (te == w.s + w.tiles);
      const int cols_here = min(NCOL, p.qH - cg * NCOL);
      const int64_t row0 = int64_t(w.b) * p.qH + int64_t(cg) * NCOL;   // first (b, i, h) row
      const int pslot = piece_slot(vc, w.s, per, p.col_groups, cg);
      if (tid < cols_here) {
        const float sum = red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
        const float lse = (sum > 0.0f && !aborted) ? (mref_s[tid] + __log2f(sum)) * kLn2 : -INFINITY;
        if (whole) p.lse[row0 + tid] = lse;
        else p.part_lse[int64_t(pslot) * NCOL + tid] = lse;
      }
      // O^T: this thread owns latent row 128*c + 32*sp + lane of every chunk c
#pragma unroll 1
      for (int n0 = 0; n0 < NCOL; n0 += 16) {
        float inv[16];
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const int col = n0 + n;
          const float sum = red[col] + red[64 + col] + red[128 + col] + red[192 + col];
          inv[n] = sum > 0.0f ? 1.0f / sum : 0.0f;
        }
        for (int c = 0; c < p.nch; ++c) {
          const int lat = 128 * c + 32 * sp + lane;
          float o[16];
          if (!aborted) {
            tmem_ld16(tmem + lane_base + (2 + c) * NCOL + n0, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int n = 0; n < 16; ++n) o[n] = 0.0f;
          }
          if (lat < p.r) {
#pragma unroll
            for (int n = 0; n < 16; ++n) {
              const int col = n0 + n;
              if (col < cols_here) {
                const float v = o[n] * inv[n];
                if (whole) p.o_latent[(row0 + col) * p.r + lat] = cvt_bf16(v);
                else p.part_o[(int64_t(pslot) * NCOL + col) * p.r + lat] = cvt_bf16(v);
              }
            }
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

#ifdef MLA_TRACE
extern "C" int mla_trace_read(unsigned long long* host, int n) {
  return int(cudaMemcpyFromSymbol(host, g_mla_trace, sizeof(unsigned long long) *
                                  size_t(n < 10 * kTraceTiles ? n : 10 * kTraceTiles)));
}
#endif


template <int NCOL>
static cudaError_t launch_decode_n(const DecodeParams& p, dim3 grid, size_t smem,
                                   cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<NCOL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_decode_kernel<NCOL>, grid, dim3(kThreads), smem, stream, 1, p);
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

}  // namespace mla
