// decode_pair.cu - mla_decode_attn on sm_100a for blocks of 65..128 query rows: a cluster
// of two CTAs splits the latent dimension.
//
// Formulation, for one block of up to 128 query rows n = (i, h) of a sequence:
//   S[n, tok]  = Q[n, :] . C[tok, :]        UMMA M=128 rows, N=64 tokens, K = row width
//   O[n, c]   += P[n, tok] C[tok, c]        UMMA M=128 rows, N=r/2 latent, K = 64 tokens
// O for 128 rows and the whole latent of rank 512 would fill all 512 TMEM columns of an
// SM, so the two CTAs of a cluster split the latent. CTA k loads, for every page, only the
// latent columns [k r/2, (k+1) r/2) and half of the rotary columns, keeps the same half of
// the Q rows in TMEM, and computes the partial scores over its half of the row width. The
// partials are swapped through distributed shared memory; both CTAs add the same two
// partials, run the same online softmax on the same numbers and so hold the same weights
// P, which each applies to its latent half. Each page crosses HBM once per cluster; Q and
// P are UMMA A operands read from TMEM, so shared-memory bandwidth goes to the cache half.
//
// The exchange. The SM-to-SM network moves about 13 bytes per clock per SM each way, so
// the partial of a tile (128 rows x 64 tokens) travels as 24-bit floats: fp32 rounded to
// a 15-bit mantissa (relative error <= 2^-16, far below the bf16 rounding of P), 4 values
// in 3 words, 24 KB per tile. Each CTA rounds its own partial the same way before adding,
// so both sides add identical numbers. Every thread sends its packed words straight from
// registers (st.async, completing on the partner's mbarrier) and keeps them for its own
// sum, so no shared memory is spent on staging and four cache slots fit. The softmax
// warps send tile j+1 before they finish tile j, so one tile of exchange latency overlaps
// the softmax and PV work of the previous tile.
//
// Roles (352 threads per CTA): warp 0 TMA producer, warp 1 S issuer and TMEM owner, warps
// 2-9 the score exchange, softmax, P into TMEM and the epilogue, warp 10 the PV issuer.
// The M=128 accumulator puts row n on TMEM lane n, and a warp reaches only the 32 lanes of
// its sub-partition (warp % 4); with 16x32bx2 TMEM accesses a warp covers 16 rows with two
// threads each (lanes i and i + 16: tokens 0-31 and 32-63 of every tile), so the row's
// maximum and sum need one shuffle, and the two warps of a sub-partition take its lanes
// 0-15 and 16-31.
//
// TMEM columns: O [0, r/2), S [256, 320), P [320, 352) (bf16 pairs), Q [352, 352 +
// (r/2 + rope_half)/2) (bf16 pairs: latent half, then rotary half).
#include <math.h>

#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

// Optional per-tile timeline of CTA 0 (compile with -DMLA_TRACE; read with
// mla_pair_trace_read). Events: 0 producer issued the tile's loads, 1 every block of the
// tile landed (the S issuer waits for that before the S buffer), 2 S committed, 3 softmax
// read S, 4 partial sent, 5 partner's partial received, 6 PV(j-1) seen done, 7 P written,
// 8 PV issued, 9 S issuer saw S free, 10 scores unpacked, 11 scores scaled. After the 12
// event rows: every CTA's start and end (%globaltimer) as pairs.
#ifdef MLA_TRACE
constexpr int kPairTraceTiles = 512;
constexpr int kPairTraceEvents = 12;
__device__ unsigned long long g_mla_pair_trace[kPairTraceEvents * kPairTraceTiles + 2 * 1024];
#define MLA_PTRACE(ev, idx)                                                              \
  do {                                                                                  \
    if (blockIdx.x == 0 && (idx) < kPairTraceTiles)                                     \
      g_mla_pair_trace[(ev) * kPairTraceTiles + (idx)] = clock64();                     \
  } while (0)
#else
#define MLA_PTRACE(ev, idx) \
  do {                     \
  } while (0)
#endif

namespace {

constexpr int kRowThreads = 2;                                   // softmax threads per row
constexpr int kSoftWarps = 8;                                  // 16 rows per warp
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kPvWarp = 2 + kSoftWarps;
constexpr int kThreads = 32 * (kPvWarp + 1);
constexpr int kQTok = kDecodeTok / kRowThreads;                  // tokens per softmax thread
constexpr uint32_t kBlk = kDecodeTok * 128;                    // 64 x 64 bf16 block, 8 KB
constexpr int kPackWords = kQTok * 3 / 4;                      // 24-bit values of one part
constexpr uint32_t kXWarpBytes = 32u * kPackWords * 4;          // one warp's parts
constexpr uint32_t kXBytes = kSoftWarps * kXWarpBytes;          // one tile's partial, 24 KB
constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352, kTmemCols = 512;
constexpr float kLazyThreshold = 8.0f;   // log2 units; see decode.cu
constexpr int kPrefetchAhead = 4;        // tiles brought into L2 ahead of their TMA load
constexpr float kRefInit = -3.0e38f;
constexpr float kLn2 = 0.69314718055994530942f;
// misc ints: 0 TMEM base, 1 abort flag, [2,8) schedule, [8, 8 + warps) warp sums
constexpr int kMiscInts = 32;

struct PairLayout {
  uint32_t slot_bytes, rope_off, recv_off, misc_off, bar_off, total;
  int nb;   // TMA barriers per slot: one per latent block and one for the rotary block
};

__host__ __device__ inline uint32_t round_up_p(uint32_t x, uint32_t a) {
  return (x + a - 1) / a * a;
}

__host__ __device__ constexpr int pair_bars(int nslot, int nb) { return nslot * nb + nslot + 10; }

__host__ __device__ inline PairLayout pair_layout(int r, int rope_half, int nslot) {
  PairLayout L;
  const int lb = r / 128;                         // 64-column latent blocks per CTA
  L.nb = lb + 1;
  L.rope_off = uint32_t(lb) * kBlk;
  L.slot_bytes = round_up_p(L.rope_off + uint32_t(kDecodeTok) * rope_half * 2, 1024);
  uint32_t off = uint32_t(nslot) * L.slot_bytes;
  L.recv_off = off;                               // partner's packed partials (two tiles)
  off += 2 * kXBytes;
  L.misc_off = off;
  off += 4 * kMiscInts;
  L.bar_off = round_up_p(off, 8);
  off = L.bar_off + 8 * pair_bars(nslot, L.nb);
  L.total = off + 1024;                           // slack for 1024-byte alignment
  return L;
}

MLA_DEVICE uint8_t* align_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

MLA_DEVICE SmemSwizzle rope_swizzle(int rope_half) {
  return rope_half == 64 ? kSw128 : (rope_half == 32 ? kSw64 : kSw32);
}

// Byte offset of 16-byte chunk c (packed words 4c..4c+3) of lane `lane` of softmax warp
// wi in a receive buffer: each warp's 32 (row, token half) threads are one contiguous
// block, chunk-major inside it, so a quarter-warp touches 128 consecutive bytes.
MLA_DEVICE uint32_t x_offset(int wi, int lane, int c) {
  return uint32_t(wi) * kXWarpBytes + uint32_t(c) * 512u + uint32_t(lane) * 16u;
}

// Four 24-bit values (fp32 rounded to sign, exponent and a 15-bit mantissa) in three words
// (value k's three bytes follow value k-1's), and back to fp32 with a zero low byte.
// Rounding adds half of the dropped byte; the byte moves are single byte permutes.
MLA_DEVICE void pack_f24(const float* v, uint32_t* w) {
  const uint32_t a = __float_as_uint(v[0]) + 0x80u, b = __float_as_uint(v[1]) + 0x80u;
  const uint32_t c = __float_as_uint(v[2]) + 0x80u, d = __float_as_uint(v[3]) + 0x80u;
  w[0] = __byte_perm(a, b, 0x5321);   // a1 a2 a3 b1
  w[1] = __byte_perm(b, c, 0x6532);   // b2 b3 c1 c2
  w[2] = __byte_perm(c, d, 0x7653);   // c3 d1 d2 d3
}
MLA_DEVICE void unpack_f24(const uint32_t* w, float* v) {
  v[0] = __uint_as_float(__byte_perm(w[0], 0u, 0x2104));
  v[1] = __uint_as_float(__byte_perm(w[0], w[1], 0x5433) & 0xFFFFFF00u);
  v[2] = __uint_as_float(__byte_perm(w[1], w[2], 0x4322) & 0xFFFFFF00u);
  v[3] = __uint_as_float(w[2] & 0xFFFFFF00u);
}

// 16x32bx2 TMEM accesses: a warp reaches 16 lanes (rows) of its sub-partition; threads
// 0-15 take columns [c, c + N) of those lanes and threads 16-31 columns [c + split,
// c + split + N), so the two threads i and i + 16 share row i.
MLA_DEVICE void tm_ld_x32_s32(uint32_t taddr, float* v) {   // N 32, split 32
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
MLA_DEVICE void tm_ld_x16_s16(uint32_t taddr, float* v) {   // N 16, split 16
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
MLA_DEVICE void tm_st_x16_s16(uint32_t taddr, const uint32_t* r) {   // N 16, split 16
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
MLA_DEVICE void tm_st_x8_s8(uint32_t taddr, const uint32_t* r) {   // N 8, split 8
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], 8, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

}  // namespace

size_t decode_pair_smem_bytes(int r, int rope_half, int nslot) {
  return pair_layout(r, rope_half, nslot).total;
}

__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_pair_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_1024(smem_raw);
  const int r = p.r, rh = p.rope_half, lb = r / 128, rhalf = r / 2;
  const PairLayout lay = pair_layout(r, rh, p.nslot);
  uint8_t* slots = base;
  uint8_t* recv = base + lay.recv_off;
  int* misc = reinterpret_cast<int*>(base + lay.misc_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = misc + 1;
  int* sched = misc + 2;
  int* warp_sum = misc + 8;
  static_assert(8 + kThreads / 32 <= kMiscInts, "misc ints overflow into the mbarriers");
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + lay.bar_off);
  const int nb = lay.nb;
  uint64_t* full = bars;                               // [slot][nb]
  uint64_t* empty = full + p.nslot * nb;               // [slot]
  uint64_t* q_full = empty + p.nslot;
  uint64_t* s_full = q_full + 1;
  uint64_t* s_free = s_full + 1;
  uint64_t* pv_done = s_free + 1;
  uint64_t* recv_full = pv_done + 1;                   // [2] partner's partial landed
  uint64_t* peer_free = recv_full + 2;                 // [2] partner consumed our partial
  uint64_t* p_full = peer_free + 2;                    // P of the tile written

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = int(blockIdx.x) >> 1;
  const int cg = pair % p.col_groups;                  // row block of this cluster
  const int vc = pair / p.col_groups;                  // index among that block's clusters
  const int vgrid = int(gridDim.x >> 1) / p.col_groups;
  const uint32_t rope_bytes = uint32_t(kDecodeTok) * rh * 2;
  const WaitCtx wc{abort_flag, p.dev_error};

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nslot; ++s) {
      for (int k = 0; k < nb; ++k) mbar_init(&full[s * nb + k], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, kSoftWarps);
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftWarps);
    mbar_init(pv_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&recv_full[i], 1);
      mbar_init(&peer_free[i], kSoftWarps);
    }
    mbar_init(p_full, kSoftWarps);
    *abort_flag = 0;
    fence_mbar_init();
    // both receive buffers expect their first partial
    mbar_arrive_expect_tx(&recv_full[0], kXBytes);
    mbar_arrive_expect_tx(&recv_full[1], kXBytes);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // Both CTAs of the cluster compute the same range (same pair index).
  find_tile_range<kThreads>(p, vc, vgrid, blockIdx.x == 0, warp_sum, sched);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the partner's barriers are initialised before anything is sent to them
  cluster_sync_all();
  const uint32_t tmem = *tmem_slot;
  const int r0 = sched[2], r1 = sched[3], per = sched[4];
  const bool has_work = sched[0] >= 0 && r0 < r1;
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024)
    g_mla_pair_trace[kPairTraceEvents * kPairTraceTiles + 2 * blockIdx.x] = globaltimer_ns();
#endif

  if (warp == 0) {
    // ===================================== TMA producer ==================================
    if (has_work && elect_one()) {
      prefetch_tensormap(&p.tm_cache);
      prefetch_tensormap(&p.tm_rope);
      if (blockIdx.x == 0) *p.range_len = per;
      UnitWalk w{sched[0], sched[1]};
      // L2 prefetch walk, kPrefetchAhead tiles ahead of the loads: the few shared-memory
      // slots leave too little lead time to hide DRAM latency behind the loads alone.
      UnitWalk pf{sched[0], sched[1]};
      pf.load(p, cg);
      int pf_t = max(pf.s, r0), pf_n = 0;
      auto prefetch_upto = [&](int upto) {
        while (pf_n < upto && pf.s < r1) {
          if (pf_t >= min(pf.s + pf.tiles, r1)) {
            pf.s += pf.tiles;
            ++pf.b;
            if (pf.s >= r1) break;
            pf.load(p, cg);
            pf_t = pf.s;
          }
          const int32_t page = p.block_table[int64_t(pf.b) * p.max_pages + (pf_t - pf.s)];
          if (page >= 0 && page < p.num_pages) {
            for (int k = 0; k < lb; ++k)
              tma_prefetch_l2_2d(&p.tm_cache, int(rank) * rhalf + k * 64, page * kDecodeTok);
            tma_prefetch_l2_2d(&p.tm_rope, r + int(rank) * rh, page * kDecodeTok);
          }
          ++pf_t;
          ++pf_n;
        }
      };
      int jj = 0;
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        if (rank == 0) p.unit_start[w.u] = w.s;   // same value from every cluster
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        const int32_t* bt = p.block_table + int64_t(w.b) * p.max_pages;
        for (int t = tb; t < te; ++t, ++jj) {
          const int slot = jj % p.nslot;
          if (jj >= p.nslot && !mbar_wait(&empty[slot], ((jj / p.nslot) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int32_t page = bt[t - w.s];
          if (page < 0 || page >= p.num_pages) {
            if (p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
            page = 0;
          }
          uint8_t* sbase = slots + slot * lay.slot_bytes;
          for (int k = 0; k < lb; ++k) {
            uint64_t* fb = &full[slot * nb + k];
            mbar_arrive_expect_tx(fb, kBlk);
            tma_load_2d(sbase + k * kBlk, &p.tm_cache, int(rank) * rhalf + k * 64,
                        page * kDecodeTok, fb);
          }
          uint64_t* fb = &full[slot * nb + lb];
          mbar_arrive_expect_tx(fb, rope_bytes);
          tma_load_2d(sbase + lay.rope_off, &p.tm_rope, r + int(rank) * rh, page * kDecodeTok,
                      fb);
          // after the load: a prefetch queued ahead of it would delay it
          prefetch_upto(jj + 1 + kPrefetchAhead);
          MLA_PTRACE(0, jj);
        }
      }
      // Drain: never leave while copies into this CTA's shared memory are in flight.
      for (int j = (jj > p.nslot ? jj - p.nslot : 0); j < jj; ++j)
        for (int k = 0; k < nb; ++k)
          mbar_wait_bounded(&full[(j % p.nslot) * nb + k], (j / p.nslot) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ UMMA issuer for the partial S ==========================
    if (has_work && elect_one()) {
      const uint32_t idesc_s = make_idesc_bf16(128, kDecodeTok, 0, 0);
      const uint64_t b0 = make_sdesc(smem_u32(slots), 16, 1024, kSw128);
      const uint64_t br0 =
          make_sdesc(smem_u32(slots + lay.rope_off), 16, 8 * rh * 2, rope_swizzle(rh));
      UnitWalk w{sched[0], sched[1]};
      int jj = 0, pc = 0;
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b, ++pc) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        if (!mbar_wait(q_full, pc & 1, wc)) { ok = false; break; }
        tc_fence_after();
        for (int t = tb; ok && t < te; ++t, ++jj) {
          const int slot = jj % p.nslot;
          // every block of the tile landed, then the S accumulator free
          for (int k = 0; ok && k <= lb; ++k)
            ok = mbar_wait(&full[slot * nb + k], (jj / p.nslot) & 1, wc);
          if (!ok) break;
          MLA_PTRACE(1, jj);
          if (jj >= 1 && !mbar_wait(s_free, (jj - 1) & 1, wc)) { ok = false; break; }
          MLA_PTRACE(9, jj);
          tc_fence_after();
          const uint32_t soff = slot * lay.slot_bytes;
          for (int k = 0; k < lb; ++k) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ts(tmem + kColS, tmem + kColQ + (k * 4 + kk) * 8,
                           b0 + ((soff + k * kBlk + kk * 32) >> 4), idesc_s,
                           (k | kk) != 0 ? 1u : 0u);
          }
          for (int kk = 0; kk < rh / 16; ++kk)
            umma_bf16_ts(tmem + kColS, tmem + kColQ + (lb * 4 + kk) * 8,
                         br0 + ((soff + kk * 32) >> 4), idesc_s, 1u);
          umma_commit(s_full);
          MLA_PTRACE(2, jj);
        }
      }
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ============================== UMMA issuer for O += P C ==============================
    if (has_work && elect_one()) {
      const uint32_t idesc_o = make_idesc_bf16(128, rhalf, 0, 1);
      // B operand: the latent blocks of the slot read MN-major (latent contiguous)
      const uint64_t pb0 = make_sdesc(smem_u32(slots), kBlk, 1024, kSw128);
      UnitWalk w{sched[0], sched[1]};
      int jj = 0;
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        for (int t = tb; t < te; ++t, ++jj) {
          if (!mbar_wait(p_full, jj & 1, wc)) { ok = false; break; }
          tc_fence_after();
          // the first tile of a piece overwrites O: the previous piece's epilogue read O
          // before its warps arrived on p_full for this tile
          const bool first = (t == tb);
          const uint32_t soff = (jj % p.nslot) * lay.slot_bytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8, pb0 + ((soff + kk * 2048) >> 4),
                         idesc_o, (!first || kk > 0) ? 1u : 0u);
          umma_commit(pv_done);
          umma_commit(&empty[jj % p.nslot]);
          MLA_PTRACE(8, jj);
        }
      }
    }
    __syncwarp();
  } else if (has_work) {
    // =========== score exchange, softmax, P, epilogue (row n, half qt of a tile) ================
    const int sp = warp & 3;                  // TMEM sub-partition this warp may access
    const int wi = warp - 2;                  // softmax warp 0..7 (exchange block index)
    const int hl = wi >> 2;                   // which 16 lanes of the sub-partition
    const int qt = lane >> 4;                 // which 32 tokens of a tile / half of O
    const int n = 32 * sp + 16 * hl + (lane & 15);   // query row: lanes i and i + 16 share it
    const int tid = threadIdx.x - 64;         // 0..255
    const uint32_t trow = tmem + (uint32_t(32 * sp + 16 * hl) << 16);
    const uint32_t recv_s = smem_u32(recv);
    const uint32_t recv_r = map_to_rank(recv_s, peer);
    const uint32_t rfull_r0 = map_to_rank(smem_u32(&recv_full[0]), peer);
    const uint32_t rfull_r1 = map_to_rank(smem_u32(&recv_full[1]), peer);
    const uint32_t pfree_r0 = map_to_rank(smem_u32(&peer_free[0]), peer);
    const uint32_t pfree_r1 = map_to_rank(smem_u32(&peer_free[1]), peer);
    const float c_log2 = p.scale_log2;
    const int row = cg * kPairRows + n;       // row (i, h) of the sequence's q*H rows
    const bool row_ok = row < p.qH;
    const int qi = row / p.num_heads;
    const bool vec_out = (reinterpret_cast<uintptr_t>(p.o_latent) & 15u) == 0;

    // Q half of this thread's row into TMEM (16-element chunks dealt alternately to the
    // two threads of the row): latent half, then rotary half; zero rows past q*H. Ends
    // with this warp's arrival on q_full.
    auto load_q = [&](int b) {
      const uint16_t* q = p.q_ext + (int64_t(b) * p.qH + row) * p.D;
      // 16-element chunks: chunk c0 / 16 + qt of the row per store (two per store)
      for (int c0 = 0; c0 < rhalf + rh; c0 += 32) {
        const int e = c0 + 16 * qt;           // past the end for an odd chunk count: zeros
        const int src = e < rhalf ? int(rank) * rhalf + e : r + int(rank) * rh + (e - rhalf);
        uint32_t v[8];
        if (row_ok && e < rhalf + rh) {
          const uint4 a = *reinterpret_cast<const uint4*>(q + src);
          const uint4 bb = *reinterpret_cast<const uint4*>(q + src + 8);
          v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
          v[4] = bb.x; v[5] = bb.y; v[6] = bb.z; v[7] = bb.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = 0u;
        }
        tm_st_x8_s8(trow + kColQ + c0 / 2, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    };

    // ---- send side: the partial of the next tile of this CTA's range ----------------
    // `sw` walks the units one tile ahead of the softmax; it loads the Q of every new
    // piece as soon as the previous piece's last S has been read out of TMEM.
    UnitWalk sw{sched[0], sched[1]};
    sw.load(p, cg);
    int st_t = max(sw.s, r0);                // next tile to send (row-block tile index)
    int js = 0;                              // tiles sent so far
    // this thread's packed partial of the tile last sent (own_next) and of the tile whose
    // scores are formed now (own_cur): the own contribution never leaves the registers
    uint32_t own_next[kPackWords], own_cur[kPackWords];
    load_q(sw.b);
    auto send_next = [&]() -> bool {
      if (st_t >= min(sw.s + sw.tiles, r1)) {
        sw.s += sw.tiles;
        ++sw.b;
        if (sw.s >= r1) return false;
        sw.load(p, cg);
        st_t = sw.s;
        load_q(sw.b);
      }
      const int kb = js & 1;
      uint32_t* pw = own_next;                 // kept for this tile's own contribution
      {
        float x[kQTok];
        const bool got = __all_sync(0xffffffffu, mbar_wait(s_full, js & 1, wc));
        if (got) {
          tc_fence_after();
          tm_ld_x32_s32(trow + kColS, x);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < kQTok; ++c) x[c] = 0.0f;
        }
        if (threadIdx.x == 64) MLA_PTRACE(3, js);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);    // the S accumulator may be overwritten
#pragma unroll
        for (int g = 0; g < kQTok / 4; ++g) pack_f24(x + 4 * g, pw + 3 * g);
      }
      // Into the partner's receive buffer once the partner has consumed tile js - 2 from
      // it: stores from registers over the SM-to-SM network, each completing its bytes on
      // the partner's mbarrier.
      const bool free_ok = __all_sync(
          0xffffffffu, js < 2 || mbar_wait_cluster(&peer_free[kb], ((js - 2) >> 1) & 1, wc));
      if (free_ok) {
        const uint32_t dst = recv_r + kb * kXBytes;
        const uint32_t rb = kb ? rfull_r1 : rfull_r0;
#pragma unroll
        for (int c = 0; c < kPackWords / 4; ++c)
          st_async_v4(dst + x_offset(wi, lane, c),
                      make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]), rb);
      }
      if (threadIdx.x == 64) MLA_PTRACE(4, js);
      ++js;
      ++st_t;
      return true;
    };

    bool sending = send_next();              // tile 0 (the range is not empty)
    UnitWalk w{sched[0], sched[1]};
    w.load(p, cg);
    int jj = 0;
    while (true) {
      const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
      const int L = w.L;
      // last position row n sees (causal: L - q + i); rows past q*H see L - 1
      const int lim = min(L - 1, p.causal ? L - p.q_len + qi : L - 1);
      float m = kRefInit, l = 0.0f;          // m identical in the two threads of a row
      for (int t = tb; t < te; ++t, ++jj) {
        const int kb = jj & 1;                 // receive buffer of this tile
        const int slot = jj % p.nslot;
        const int tile_pos0 = (t - w.s) * kDecodeTok;
        const int pos0 = tile_pos0 + qt * kQTok;   // first token of this thread's half
        // ---- send the next tile's partial before finishing this one ----
#pragma unroll
        for (int i = 0; i < kPackWords; ++i) own_cur[i] = own_next[i];
        if (sending) sending = send_next();
        // ---- this tile's scores: own rounded partial + the partner's ----
        const bool rcv =
            __all_sync(0xffffffffu, mbar_wait_cluster(&recv_full[kb], (jj >> 1) & 1, wc));
        if (threadIdx.x == 64) MLA_PTRACE(5, jj);
        float s[kQTok];
        {
          const uint32_t oth = recv_s + kb * kXBytes;
          uint32_t wb[kPackWords];
#pragma unroll
          for (int c = 0; c < kPackWords / 4; ++c) {
            const uint4 vb = ld_shared_v4(oth + x_offset(wi, lane, c));
            wb[4 * c] = vb.x; wb[4 * c + 1] = vb.y; wb[4 * c + 2] = vb.z; wb[4 * c + 3] = vb.w;
          }
#pragma unroll
          for (int g = 0; g < kQTok / 4; ++g) {
            float fa[4], fb[4];
            unpack_f24(own_cur + 3 * g, fa);
            unpack_f24(wb + 3 * g, fb);
#pragma unroll
            for (int i = 0; i < 4; ++i) s[4 * g + i] = rcv ? fa[i] + fb[i] : 0.0f;
          }
        }
        if (threadIdx.x == 64) MLA_PTRACE(10, jj);
        __syncwarp();
        // The received words are in registers (consumed above): release the buffer to the
        // partner without a release fence, which would wait for this warp's remote stores.
        if (lane == 1) mbar_arrive_remote_relaxed(kb ? pfree_r1 : pfree_r0);
        // re-arm this buffer for tile jj + 2 (the partner sends it only after all eight
        // warps have released the buffer above)
        if (threadIdx.x == 65 && rcv) mbar_arrive_expect_tx_relaxed(&recv_full[kb], kXBytes);

        // ---- online softmax of row n over this tile (log2 domain, lazy reference) ----
        if (pos0 + kQTok - 1 > lim) {
#pragma unroll
          for (int c = 0; c < kQTok; ++c)
            if (pos0 + c > lim) s[c] = -INFINITY;
        }
        // maximum of the raw scores (a tree; the positive scale is applied once after it)
        float mt[kQTok / 2];
#pragma unroll
        for (int c = 0; c < kQTok / 2; ++c) mt[c] = fmaxf(s[c], s[c + kQTok / 2]);
#pragma unroll
        for (int w2 = kQTok / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int c = 0; c < w2; ++c) mt[c] = fmaxf(mt[c], mt[c + w2]);
        // the row's maximum over both halves (lanes i and i + 16: the same value in both)
        const float mh = mt[0] * c_log2;
        const float mx = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
        if (threadIdx.x == 64) MLA_PTRACE(11, jj);
        float alpha = 1.0f;
        if (mx > m + kLazyThreshold) {
          alpha = ex2_approx(m - mx);          // 0 while m is still kRefInit
          l *= alpha;
          m = mx;
        }
        // PV(jj-1) reads P and accumulates into O: wait for it before touching either
        const bool pv_ok =
            __all_sync(0xffffffffu, jj == 0 || mbar_wait(pv_done, (jj - 1) & 1, wc));
        if (threadIdx.x == 64) MLA_PTRACE(6, jj);
        tc_fence_after();
        if (t > tb && pv_ok && __any_sync(0xffffffffu, alpha != 1.0f)) {
          for (int c0 = 0; c0 < rhalf; c0 += 32) {
            float o[16];
            tm_ld_x16_s16(trow + kColO + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] *= alpha;
            tm_st_x16_s16(trow + kColO + c0, reinterpret_cast<const uint32_t*>(o));
          }
        }
        // weights 2^(s * scale - m); the tile's sum in two chains, added to l in a fixed
        // order (both CTAs of the pair agree bit for bit)
        uint32_t pk[kQTok / 2];
        float sa = 0.0f, sb = 0.0f;
#pragma unroll
        for (int c = 0; c < kQTok / 2; ++c) {
          const float p0 = ex2_approx(fmaf(s[2 * c], c_log2, -m));
          const float p1 = ex2_approx(fmaf(s[2 * c + 1], c_log2, -m));
          sa += p0;
          sb += p1;
          pk[c] = cvt_bf16x2(p0, p1);
        }
        l += sa + sb;
        tm_st_x16_s16(trow + kColP, pk);
        // cache rows past the context may hold anything (even NaN): zero their latent half
        // so that 0-weight x garbage cannot reach O
        if (tile_pos0 + kDecodeTok > L) {
          const int tok = tid & (kDecodeTok - 1);
          if (tile_pos0 + tok >= L) {
            uint8_t* sbase = slots + slot * lay.slot_bytes;
            for (int k = tid >> 6; k < lb; k += kSoftThreads / kDecodeTok) {
              uint4* rowp = reinterpret_cast<uint4*>(sbase + k * kBlk + tok * 128);
#pragma unroll
              for (int ch = 0; ch < 8; ++ch) rowp[ch] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        // P (and any O rescale and zeroed rows) complete: hand the tile to the PV issuer
        tmem_wait_st();
        if (threadIdx.x == 64) MLA_PTRACE(7, jj);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }

      // ---------------------------- epilogue of this piece --------------------------------
      const bool fin = __all_sync(0xffffffffu, mbar_wait(pv_done, (jj - 1) & 1, wc));
      tc_fence_after();
      const bool aborted = __any_sync(0xffffffffu, !fin || *abort_flag != 0);
      // the row sum over both halves (the same value in both threads: a + b = b + a)
      const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const bool whole = (tb == w.s) && (te == w.s + w.tiles);
      const int64_t grow = int64_t(w.b) * p.qH + row;   // global (b, i, h) row
      const int pslot = piece_slot(vc, w.s, per, p.col_groups, cg);
      const float lse = (lt > 0.0f && !aborted) ? (m + __log2f(lt)) * kLn2 : -INFINITY;
      if (row_ok && rank == 0 && qt == 0) {
        if (whole) p.lse[grow] = lse;
        else p.part_lse[int64_t(pslot) * kPairRows + n] = lse;
      }
      const float inv = (lt > 0.0f && !aborted) ? 1.0f / lt : 0.0f;
      const int64_t lat0 = int64_t(rank) * rhalf + 16 * qt;   // this thread's 16 of every 32
      for (int c0 = 0; c0 < rhalf; c0 += 32) {
        float o[16];
        if (!aborted) {
          tm_ld_x16_s16(trow + kColO + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] = 0.0f;
        }
        if (!row_ok) {
          // padding row past q*H: nothing to write
        } else if (whole) {
          uint16_t* dst = p.o_latent + grow * r + lat0 + c0;
          if (vec_out) {
#pragma unroll
            for (int c = 0; c < 16; c += 8)
              *reinterpret_cast<uint4*>(dst + c) =
                  make_uint4(cvt_bf16x2(o[c] * inv, o[c + 1] * inv),
                             cvt_bf16x2(o[c + 2] * inv, o[c + 3] * inv),
                             cvt_bf16x2(o[c + 4] * inv, o[c + 5] * inv),
                             cvt_bf16x2(o[c + 6] * inv, o[c + 7] * inv));
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) dst[c] = f32_to_bf16_rne(o[c] * inv);
          }
        } else {
          float* dst = p.part_o + (int64_t(pslot) * kPairRows + n) * r + lat0 + c0;
#pragma unroll
          for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
        }
      }
      tc_fence_before();
      w.s += w.tiles;
      ++w.b;
      if (w.s >= r1) break;
      w.load(p, cg);
    }
  }

  tc_fence_before();
  __syncthreads();
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024)
    g_mla_pair_trace[kPairTraceEvents * kPairTraceTiles + 2 * blockIdx.x + 1] = globaltimer_ns();
#endif
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  // neither CTA leaves while its partner may still write into its shared memory
  cluster_sync_all();
}

#ifdef MLA_TRACE
extern "C" int mla_pair_trace_read(unsigned long long* host, int n) {
  const int cap = kPairTraceEvents * kPairTraceTiles + 2 * 1024;
  return int(cudaMemcpyFromSymbol(host, g_mla_pair_trace,
                                  sizeof(unsigned long long) * size_t(n < cap ? n : cap)));
}
#endif

int decode_pair_max_clusters(size_t smem) {
  if (cudaFuncSetAttribute(mla_decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, mla_decode_pair_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_decode_pair(const DecodeParams& p, dim3 grid, size_t smem,
                               cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_pair_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, mla_decode_pair_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
