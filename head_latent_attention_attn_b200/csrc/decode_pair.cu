// decode_pair.cu - mla_decode_attn on sm_100a for blocks of 65..128 query rows: a cluster
// of two CTAs splits the latent dimension and shares the softmax by rows.
//
// Formulation, for one block of up to 128 query rows n = (i, h) of a sequence:
//   S[n, tok]  = Q[n, :] . C[tok, :]        UMMA M=128 rows, N=64 tokens, K = row width
//   O[n, c]   += P[n, tok] C[tok, c]        UMMA M=128 rows, N=r/2 latent, K = 64 tokens
// O for 128 rows and the whole latent of rank 512 would fill all 512 TMEM columns of an
// SM, so the two CTAs of a cluster split the latent. CTA k loads, for every page, only the
// latent columns [k r/2, (k+1) r/2) and half of the rotary columns, keeps the same half of
// every Q row, and computes the partial scores S_k over its half of the row width. Each
// page crosses HBM once per cluster.
//
// The softmax is split by rows. CTA k owns 64 of the 128 rows: it receives the partner's
// partial scores for those rows only, adds them to its own, runs the online softmax and
// writes P for its rows into its TMEM; it also sends those weights (bf16), with the row's
// rescale factor and running sum, to the partner, whose O half needs P for all 128 rows.
// Per tile and direction that is 12 KB of partial scores (24-bit floats: fp32 rounded to
// a 15-bit mantissa, relative error <= 2^-16, 4 values in 3 words) and 8.5 KB of weights,
// and each CTA evaluates 64 x 64 exponentials instead of 128 x 64.
//
// TMEM (512 columns): O [0, r/2), two S buffers [256, 320) and [320, 384), two P buffers
// (bf16 pairs) [384, 416) and [416, 448), and the first 128 latent elements of Q [448, 512)
// (bf16 pairs). The rest of Q's latent half and its rotary half are shared-memory UMMA
// operands (the S UMMA takes A from TMEM for the first K steps and from shared memory for
// the others). With P in its own buffers, S of tile j + 2 waits only until the scores of
// tile j have been read, not for PV of tile j.
//
// Roles (480 threads): warp 0 TMA producer, warp 1 S issuer and TMEM owner, warp 2 PV
// issuer, warps 3-14 the rows. TMEM lane n holds row n and a warp reaches only the 32 lanes
// of its sub-partition (warp % 4). CTA k owns the rows on lanes 16k..16k+15 of every
// sub-partition, so each of the three row roles has one warp on every SM sub-partition
// (its issue slots and MUFU units). With 16x32bx2 TMEM accesses a warp covers 16 lanes,
// two threads per row (lanes i and i + 16: tokens 0-31 and 32-63):
//   owners    (warps 3-6, this CTA's rows): combine the two partials, softmax, P, the
//              epilogue and lse of the own rows;
//   senders   (warps 7-10, the partner's rows): read their partial scores and send them;
//   receivers (warps 11-14, the partner's rows): take the partner's P and rescale factors
//              for those rows into TMEM, and their epilogue.
#include <math.h>

#include "decode_sched.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace mla {

// Optional per-tile timeline of CTA 0 (compile with -DMLA_TRACE; read with
// mla_pair_trace_read). Events: 0 producer issued the tile's loads, 1 every block of the
// tile landed, 2 S committed, 3 sender read S, 4 sender's partial sent, 5 owner has the
// partner's partial, 6 owner's P written and sent, 7 receiver has the partner's P, 8 PV
// issued, 9 S issuer saw the S buffer free, 10 owner read S, 11 receiver's P written.
// After the 12 event rows: every CTA's start and end (%globaltimer) as pairs.
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

constexpr int kPvWarp = 2;
constexpr int kRowWarp0 = 3;                                   // first of the 12 row warps
constexpr int kThreads = 32 * (kRowWarp0 + 12);
constexpr int kHalfTok = kDecodeTok / 2;                       // tokens per owner thread
constexpr uint32_t kBlk = kDecodeTok * 128;                    // 64 x 64 bf16 block, 8 KB
constexpr int kPackWords = kHalfTok * 3 / 4;                   // 24-bit values of a half row
constexpr uint32_t kXsWarpBytes = 32u * kPackWords * 4;        // one owner warp's rows
constexpr uint32_t kXsBytes = 4 * kXsWarpBytes;                // partials of 64 rows, 12 KB
constexpr uint32_t kXpRowsBytes = 64u * kDecodeTok * 2;        // P of 64 rows (bf16), 8 KB
constexpr uint32_t kXpBytes = kXpRowsBytes + 64u * 8;          // + (alpha, sum) per row
constexpr uint32_t kColO = 0, kColS = 256, kColP = 384, kColQ = 448, kTmemCols = 512;
constexpr int kQTmem = 128;   // latent elements of each Q row held in TMEM (the rest: smem)
constexpr float kLazyThreshold = 8.0f;   // log2 units; see decode.cu
constexpr float kRefInit = -3.0e38f;
constexpr float kLn2 = 0.69314718055994530942f;
// misc ints: 0 TMEM base, 1 abort flag, [2,8) schedule, [8, 8 + warps) warp sums
constexpr int kMiscInts = 32;

struct PairLayout {
  uint32_t slot_bytes, rope_off, qrope_off, qlat_off, xs_off, xp_off, misc_off, bar_off, total;
};

__host__ __device__ inline uint32_t round_up_p(uint32_t x, uint32_t a) {
  return (x + a - 1) / a * a;
}

__host__ __device__ constexpr int pair_bars(int nslot) { return 2 * nslot + 16; }

__host__ __device__ inline PairLayout pair_layout(int r, int rope_half, int nslot) {
  PairLayout L;
  const int lb = r / 128;                         // 64-column latent blocks per CTA
  L.rope_off = uint32_t(lb) * kBlk;
  L.slot_bytes = round_up_p(L.rope_off + uint32_t(kDecodeTok) * rope_half * 2, 1024);
  uint32_t off = uint32_t(nslot) * L.slot_bytes;
  L.qrope_off = off;                              // rotary half of the 128 Q rows (swizzled)
  off += round_up_p(uint32_t(kPairRows) * rope_half * 2, 1024);
  L.qlat_off = off;                               // latent Q past kQTmem, 64-column blocks
  off += uint32_t(kPairRows) * uint32_t(r / 2 > kQTmem ? r / 2 - kQTmem : 0) * 2;
  L.xs_off = off;                                 // partner's partials for the own rows (x2)
  off += 2 * kXsBytes;
  L.xp_off = off;                                 // partner's P for its rows
  off += kXpBytes;
  L.misc_off = off;
  off += 4 * kMiscInts;
  L.bar_off = round_up_p(off, 8);
  off = L.bar_off + 8 * pair_bars(nslot);
  L.total = off + 1024;                           // slack for 1024-byte alignment
  return L;
}

MLA_DEVICE uint8_t* align_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

MLA_DEVICE SmemSwizzle rope_swizzle(int rope_half) {
  return rope_half == 64 ? kSw128 : (rope_half == 32 ? kSw64 : kSw32);
}

// Byte offset, in a partial-score buffer, of 16-byte chunk c (packed words 4c..4c+3) for
// lane `lane` of owner warp ow: each owner warp's 32 (row, token half) threads are one
// contiguous block, chunk-major inside it, so a quarter-warp touches 128 consecutive bytes.
MLA_DEVICE uint32_t xs_offset(int ow, int lane, int c) {
  return uint32_t(ow) * kXsWarpBytes + uint32_t(c) * 512u + uint32_t(lane) * 16u;
}

// Byte offset of 16-byte chunk c (tokens 8c..8c+7, bf16) of own-block row m (0..63) in a
// weight buffer: chunk-major, so the 32 rows a receiver warp reads are consecutive; the
// rows' (alpha, running sum) pairs follow the weights.
MLA_DEVICE uint32_t xp_offset(int m, int c) { return uint32_t(c) * 1024u + uint32_t(m) * 16u; }
MLA_DEVICE uint32_t xp_scalars(int m) { return kXpRowsBytes + uint32_t(m) * 8u; }

// Byte offset of 16-byte chunk c of row `row` in a K-major tile with rows of `pitch` bytes
// (32, 64 or 128) stored with the matching 32/64/128-byte swizzle: the chunk index is
// XORed with bits 7.. of the linear offset (the layout TMA writes and UMMA reads).
MLA_DEVICE uint32_t swizzled_chunk(int row, int c, int pitch) {
  const uint32_t lin = uint32_t(row) * uint32_t(pitch) + uint32_t(c) * 16u;
  const uint32_t mask = uint32_t(pitch / 16 - 1);
  return lin ^ (((lin >> 7) & mask) << 4);
}

// Latent Q elements [e, e + 16) of row n (e a multiple of 16, counted from the first element
// past the TMEM part) into the shared-memory A operand: 64-element K-major blocks of 128 rows,
// 128-byte swizzle (the layout the S UMMA's descriptor reads).
MLA_DEVICE void store_qlat(uint8_t* qlat, int n, int e, const uint32_t* v) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int el = e + 8 * i;
    const uint32_t off = uint32_t(el / 64) * (kPairRows * 128) + uint32_t(n) * 128 +
                         ((uint32_t((el % 64) / 8) ^ uint32_t(n & 7)) << 4);
    *reinterpret_cast<uint4*>(qlat + off) =
        make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

MLA_DEVICE void st_async_v2(uint32_t remote_addr, uint2 v, uint32_t remote_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];"
      ::"r"(remote_addr), "r"(v.x), "r"(v.y), "r"(remote_bar)
      : "memory");
}
MLA_DEVICE uint2 ld_shared_v2(uint32_t saddr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(saddr) : "memory");
  return v;
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
  uint8_t* qrope = base + lay.qrope_off;
  uint8_t* qlat = base + lay.qlat_off;
  uint8_t* xs = base + lay.xs_off;
  uint8_t* xp = base + lay.xp_off;
  int* misc = reinterpret_cast<int*>(base + lay.misc_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = misc + 1;
  int* sched = misc + 2;
  int* warp_sum = misc + 8;
  static_assert(8 + kThreads / 32 <= kMiscInts, "misc ints overflow into the mbarriers");
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + lay.bar_off);
  // One barrier per slot for all of a page's TMA boxes: the S issuer needs every box before
  // it starts, and each mbarrier operation here costs a few hundred cycles of latency.
  uint64_t* full = bars;                               // [slot]
  uint64_t* empty = full + p.nslot;                    // [slot]
  uint64_t* q_full = empty + p.nslot;                  // Q of the piece in TMEM and smem
  uint64_t* s_full = q_full + 1;                       // [2] S buffer computed
  uint64_t* s_free = s_full + 2;                       // [2] S buffer read by all readers
  uint64_t* pv_done = s_free + 2;                      // [2] PV of the buffer's tile done
  uint64_t* p_full = pv_done + 2;                      // [2] P of all 128 rows written
  uint64_t* xs_full = p_full + 2;                      // [2] partner's partials landed
  uint64_t* xs_free = xs_full + 2;                     // [2] partner consumed ours
  uint64_t* xp_full = xs_free + 2;                     // partner's P landed
  uint64_t* xp_free = xp_full + 1;                     // partner consumed our P

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
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 8);                              // 4 owner + 4 sender warps
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 8);                        // 4 owner + 4 sender warps
      mbar_init(&pv_done[i], 1);
      mbar_init(&p_full[i], 8);                        // 4 owner + 4 receiver warps
      mbar_init(&xs_full[i], 1);
      mbar_init(&xs_free[i], 4);                       // the partner's 4 owner warps
    }
    mbar_init(xp_full, 1);
    mbar_init(xp_free, 4);                             // the partner's 4 receiver warps
    *abort_flag = 0;
    fence_mbar_init();
    // the receive buffers expect their first messages
    mbar_arrive_expect_tx(&xs_full[0], kXsBytes);
    mbar_arrive_expect_tx(&xs_full[1], kXsBytes);
    mbar_arrive_expect_tx(xp_full, kXpBytes);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // set-up above may overlap the previous kernel; from here on global memory is touched
  grid_dep_wait();
  grid_dep_launch();
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
      int jj = 0;
      SlotRing ring(p.nslot);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        if (rank == 0) p.unit_start[w.u] = w.s;   // same value from every cluster
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        const int32_t* bt = p.block_table + int64_t(w.b) * p.max_pages;
        for (int t = tb; t < te; ++t, ++jj, ring.next()) {
          const int slot = ring.slot;
          // the page id is read before the wait, so its round trip overlaps it
          int32_t page = bt[t - w.s];
          if (jj >= p.nslot && !mbar_wait(&empty[slot], (ring.round - 1) & 1, wc)) {
            ok = false;
            break;
          }
          if (page < 0 || page >= p.num_pages) {
            if (p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
            page = 0;
          }
          uint8_t* sbase = slots + slot * lay.slot_bytes;
          uint64_t* fb = &full[slot];
          mbar_arrive_expect_tx(fb, uint32_t(lb) * kBlk + rope_bytes);
          for (int k = 0; k < lb; ++k)
            tma_load_2d(sbase + k * kBlk, &p.tm_cache, int(rank) * rhalf + k * 64,
                        page * kDecodeTok, fb);
          tma_load_2d(sbase + lay.rope_off, &p.tm_rope, r + int(rank) * rh, page * kDecodeTok,
                      fb);
          MLA_PTRACE(0, jj);
        }
      }
      // Drain: never leave while copies into this CTA's shared memory are in flight.
      for (int j = (jj > p.nslot ? jj - p.nslot : 0); j < jj; ++j)
        mbar_wait_bounded(&full[j % p.nslot], (j / p.nslot) & 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ UMMA issuer for the partial S ==========================
    // S of tile j goes to buffer j % 2: it waits for its page and for the readers of tile
    // j - 2's scores (P has buffers of its own).
    if (has_work && elect_one()) {
      const uint32_t idesc_s = make_idesc_bf16(128, kDecodeTok, 0, 0);
      const uint64_t b0 = make_sdesc(smem_u32(slots), 16, 1024, kSw128);
      const uint64_t br0 =
          make_sdesc(smem_u32(slots + lay.rope_off), 16, 8 * rh * 2, rope_swizzle(rh));
      const uint64_t aq0 = make_sdesc(smem_u32(qrope), 16, 8 * rh * 2, rope_swizzle(rh));
      const uint64_t aql0 = make_sdesc(smem_u32(qlat), 16, 1024, kSw128);
      const int kt = 4 * (min(rhalf, kQTmem) / 64);   // latent K steps with A in TMEM
      UnitWalk w{sched[0], sched[1]};
      int jj = 0, pc = 0;
      SlotRing ring(p.nslot);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b, ++pc) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        if (!mbar_wait(q_full, pc & 1, wc)) { ok = false; break; }
        tc_fence_after();
        for (int t = tb; ok && t < te; ++t, ++jj, ring.next()) {
          const int slot = ring.slot;
          const int sb = jj & 1;
          // every block of the tile landed, then the S buffer free
          if (!mbar_wait(&full[slot], ring.round & 1, wc)) { ok = false; break; }
          MLA_PTRACE(1, jj);
          if (jj >= 2 && !mbar_wait(&s_free[sb], ((jj - 2) >> 1) & 1, wc)) {
            ok = false;
            break;
          }
          MLA_PTRACE(9, jj);
          tc_fence_after();
          const uint32_t dS = tmem + kColS + 64 * sb;
          const uint32_t soff = slot * lay.slot_bytes;
          // latent K steps: A = Q from TMEM (8 columns per step) for the first kt steps and
          // from shared memory after them; B steps 32 bytes within a 64-column block and to
          // the next block after its fourth step; then the rotary steps
          {
            uint64_t bd = b0 + (soff >> 4);
            umma_bf16_ts(dS, tmem + kColQ, bd, idesc_s, 0u);
            for (int i = 1; i < kt; ++i) {
              bd += (i & 3) == 0 ? uint64_t((kBlk - 96) >> 4) : uint64_t(2);
              umma_bf16_ts(dS, tmem + kColQ + i * 8, bd, idesc_s, 1u);
            }
            uint64_t qd = aql0;
            for (int i = kt; i < 4 * lb; ++i) {
              bd += (i & 3) == 0 ? uint64_t((kBlk - 96) >> 4) : uint64_t(2);
              if (i > kt) qd += (i & 3) == 0 ? uint64_t(((kPairRows * 128) - 96) >> 4) : uint64_t(2);
              umma_bf16(dS, qd, bd, idesc_s, 1u);
            }
            uint64_t ad = aq0, rd = br0 + (soff >> 4);
            for (int kk = 0; kk < rh / 16; ++kk, ad += 2, rd += 2) umma_bf16(dS, ad, rd, idesc_s, 1u);
          }
          umma_commit(&s_full[sb]);
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
      SlotRing ring(p.nslot);
      bool ok = true;
      for (; ok && w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        for (int t = tb; t < te; ++t, ++jj, ring.next()) {
          const int sb = jj & 1;
          if (!mbar_wait(&p_full[sb], (jj >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          // the first tile of a piece overwrites O: the previous piece's epilogue read O
          // before its warps arrived on p_full for this tile
          const bool first = (t == tb);
          const uint32_t soff = ring.slot * lay.slot_bytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tmem + kColO, tmem + kColP + 32 * sb + kk * 8,
                         pb0 + ((soff + kk * 2048) >> 4), idesc_o,
                         (!first || kk > 0) ? 1u : 0u);
          umma_commit(&pv_done[sb]);
          umma_commit(&empty[ring.slot]);
          MLA_PTRACE(8, jj);
        }
      }
    }
    __syncwarp();
  } else if (has_work) {
    // ==================================== the 128 rows ====================================
    // Every row warp works on 16 TMEM lanes of its sub-partition with 16x32bx2 accesses:
    // lanes i and i + 16 of the warp share row i and take tokens 0-31 and 32-63 (or the
    // two 16-column halves of every 32 columns of O).
    const int sp = warp & 3;                  // TMEM sub-partition this warp reaches
    const int role = (warp - kRowWarp0) >> 2; // 0 owner, 1 sender, 2 receiver
    const int qt = lane >> 4;                 // token half of this thread
    const int i16 = lane & 15;
    // owners work on this CTA's rows, senders and receivers on the partner's
    const uint32_t grp = uint32_t(32 * sp + 16 * int(role == 0 ? rank : peer));
    const int n = int(grp) + i16;             // query row (TMEM lane)
    const int m = 16 * sp + i16;              // row within its CTA's block of 64
    const uint32_t trow = tmem + (grp << 16);
    const int row = cg * kPairRows + n;       // row (i, h) of the sequence's q*H rows
    const bool row_ok = row < p.qH;
    const float c_log2 = p.scale_log2;
    const bool vec_out = (reinterpret_cast<uintptr_t>(p.o_latent) & 15u) == 0;
    const int rpitch = rh * 2;                // bytes per Q rotary row in shared memory
    const bool tr = (sp == 0 && lane == 0);
    (void)tr;
    const uint32_t xs_s = smem_u32(xs), xp_s = smem_u32(xp);
    const uint32_t xs_r = map_to_rank(xs_s, peer), xp_r = map_to_rank(xp_s, peer);
    const uint32_t xs_full_r0 = map_to_rank(smem_u32(&xs_full[0]), peer);
    const uint32_t xs_full_r1 = map_to_rank(smem_u32(&xs_full[1]), peer);
    const uint32_t xs_free_r0 = map_to_rank(smem_u32(&xs_free[0]), peer);
    const uint32_t xs_free_r1 = map_to_rank(smem_u32(&xs_free[1]), peer);
    const uint32_t xp_full_r = map_to_rank(smem_u32(xp_full), peer);
    const uint32_t xp_free_r = map_to_rank(smem_u32(xp_free), peer);

    // This CTA's half of Q row n: the latent half into TMEM (16-element chunks dealt
    // alternately to the two threads of the row), the rotary half into shared memory;
    // zero rows past q*H. Ends with this warp's arrival on q_full (owners and senders).
    auto load_q = [&](int b) {
      const uint16_t* q = p.q_ext + (int64_t(b) * p.qH + row) * p.D;
      for (int c0 = 0; c0 < rhalf; c0 += 32) {
        const uint16_t* src = q + int(rank) * rhalf + c0 + 16 * qt;
        uint32_t v[8];
        if (row_ok) {
          const uint4 a = *reinterpret_cast<const uint4*>(src);
          const uint4 bb = *reinterpret_cast<const uint4*>(src + 8);
          v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
          v[4] = bb.x; v[5] = bb.y; v[6] = bb.z; v[7] = bb.w;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = 0u;
        }
        if (c0 < kQTmem) tm_st_x8_s8(trow + kColQ + c0 / 2, v);
        else store_qlat(qlat, n, c0 + 16 * qt - kQTmem, v);
      }
      for (int c = qt; c < rh / 8; c += 2) {
        const uint4 v = row_ok ? *reinterpret_cast<const uint4*>(q + r + int(rank) * rh + 8 * c)
                               : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(qrope + swizzled_chunk(n, c, rpitch)) = v;
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    };

    // O rows of this warp times alpha (16 of every 32 columns per thread), once PV(jj - 1)
    // has landed in O.
    auto rescale_o = [&](int jj, float alpha) {
      const bool pv_ok =
          __all_sync(0xffffffffu, mbar_wait(&pv_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, wc));
      tc_fence_after();
      if (!pv_ok) return;
      for (int c0 = 0; c0 < rhalf; c0 += 32) {
        float o[16];
        tm_ld_x16_s16(trow + kColO + c0, o);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] *= alpha;
        tm_st_x16_s16(trow + kColO + c0, reinterpret_cast<const uint32_t*>(o));
      }
    };

    // O rows of this warp divided by the row sum lt, to the outputs of piece (w, tb, te)
    // whose last tile is jl: bf16 o_latent when the piece is the whole unit, else the bf16 partial part_o.
    auto write_o = [&](const UnitWalk& w, int tb, int te, int jl, float lt, bool* aborted_out) {
      const bool fin = __all_sync(0xffffffffu, mbar_wait(&pv_done[jl & 1], (jl >> 1) & 1, wc));
      tc_fence_after();
      const bool aborted = __any_sync(0xffffffffu, !fin || *abort_flag != 0);
      *aborted_out = aborted;
      const bool whole = (tb == w.s) && (te == w.s + w.tiles);
      const int64_t grow = int64_t(w.b) * p.qH + row;   // global (b, i, h) row
      const int pslot = piece_slot(vc, w.s, per, p.col_groups, cg);
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
          // bf16 partial (16-byte aligned: r % 8 == 0 and lat0 + c0 a multiple of 16)
          uint16_t* dst = p.part_o + (int64_t(pslot) * kPairRows + n) * r + lat0 + c0;
#pragma unroll
          for (int c = 0; c < 16; c += 8)
            *reinterpret_cast<uint4*>(dst + c) =
                make_uint4(cvt_bf16x2(o[c] * inv, o[c + 1] * inv),
                           cvt_bf16x2(o[c + 2] * inv, o[c + 3] * inv),
                           cvt_bf16x2(o[c + 4] * inv, o[c + 5] * inv),
                           cvt_bf16x2(o[c + 6] * inv, o[c + 7] * inv));
        }
      }
      tc_fence_before();
    };

    if (role == 0) {
      // ------------- owner: this CTA's 16 rows of sub-partition sp; softmax and P ---------
      const int qi = row / p.num_heads;
      load_q(sched[0]);
      UnitWalk w{sched[0], sched[1]};
      w.load(p, cg);
      int jj = 0;
      SlotRing ring(p.nslot);
      while (true) {
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        const int L = w.L;
        // last position row n sees (causal: L - q + i); rows past q*H see L - 1
        const int lim = min(L - 1, p.causal ? L - p.q_len + qi : L - 1);
        float mref = kRefInit, l = 0.0f, lt = 0.0f;   // the same in both threads of a row
        for (int t = tb; t < te; ++t, ++jj, ring.next()) {
          const int sb = jj & 1;                 // S buffer and partial buffer of this tile
          const int slot = ring.slot;
          const int tile_pos0 = (t - w.s) * kDecodeTok;
          const int pos0 = tile_pos0 + qt * kHalfTok;   // first token of this thread's half
          // ---- own partial scores ----
          float s[kHalfTok];
          const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (jj >> 1) & 1, wc));
          tc_fence_after();
          if (got) {
            tm_ld_x32_s32(trow + kColS + 64 * sb, s);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < kHalfTok; ++c) s[c] = 0.0f;
          }
          if (tr) MLA_PTRACE(10, jj);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[sb]);
          // S of the piece's last tile is complete: the next piece's Q may replace this one
          if (t == te - 1 && w.s + w.tiles < r1) load_q(w.b + 1);
          // ---- plus the partner's partial ----
          const bool rcv =
              __all_sync(0xffffffffu, mbar_wait_cluster(&xs_full[sb], (jj >> 1) & 1, wc));
          if (tr) MLA_PTRACE(5, jj);
          {
            const uint32_t src = xs_s + sb * kXsBytes;
            uint32_t wb[kPackWords];
#pragma unroll
            for (int c = 0; c < kPackWords / 4; ++c) {
              const uint4 v = ld_shared_v4(src + xs_offset(sp, lane, c));
              wb[4 * c] = v.x; wb[4 * c + 1] = v.y; wb[4 * c + 2] = v.z; wb[4 * c + 3] = v.w;
            }
#pragma unroll
            for (int g = 0; g < kHalfTok / 4; ++g) {
              float f[4];
              unpack_f24(wb + 3 * g, f);
#pragma unroll
              for (int k = 0; k < 4; ++k) s[4 * g + k] = rcv ? s[4 * g + k] + f[k] : 0.0f;
            }
          }
          __syncwarp();
          // The received words are in registers: release the buffer to the partner without a
          // release fence (which would wait for this warp's remote stores), and re-arm it for
          // tile jj + 2 (the partner sends that only after all four owner warps released it).
          if (lane == 1) mbar_arrive_remote_relaxed(sb ? xs_free_r1 : xs_free_r0);
          if (sp == 0 && lane == 0 && rcv) mbar_arrive_expect_tx_relaxed(&xs_full[sb], kXsBytes);

          // ---- online softmax of row n over this tile (log2 domain, lazy reference) ----
          if (pos0 + kHalfTok - 1 > lim) {
#pragma unroll
            for (int c = 0; c < kHalfTok; ++c)
              if (pos0 + c > lim) s[c] = -INFINITY;
          }
          float mt[kHalfTok / 2];
#pragma unroll
          for (int c = 0; c < kHalfTok / 2; ++c) mt[c] = fmaxf(s[c], s[c + kHalfTok / 2]);
#pragma unroll
          for (int w2 = kHalfTok / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
            for (int c = 0; c < w2; ++c) mt[c] = fmaxf(mt[c], mt[c + w2]);
          const float mh = mt[0] * c_log2;
          const float mx = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
          float alpha = 1.0f;
          if (mx > mref + kLazyThreshold) {
            alpha = ex2_approx(mref - mx);       // 0 while mref is still kRefInit
            l *= alpha;
            mref = mx;
          }
          // O rows of an earlier tile of the piece: rescale (the first tile overwrites O)
          if (t > tb && __any_sync(0xffffffffu, alpha != 1.0f)) rescale_o(jj, alpha);
          // weights 2^(s * scale - m) over the S buffer (its scores are in registers)
          uint32_t pk[kHalfTok / 2];
          float sa = 0.0f, sc = 0.0f;
#pragma unroll
          for (int c = 0; c < kHalfTok / 2; ++c) {
            const float p0 = ex2_approx(fmaf(s[2 * c], c_log2, -mref));
            const float p1 = ex2_approx(fmaf(s[2 * c + 1], c_log2, -mref));
            sa += p0;
            sc += p1;
            pk[c] = cvt_bf16x2(p0, p1);
          }
          l += sa + sc;
          lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
          if (jj >= 2) {
            __all_sync(0xffffffffu, mbar_wait(&pv_done[sb], ((jj - 2) >> 1) & 1, wc));
            tc_fence_after();
          }
          tm_st_x16_s16(trow + kColP + 32 * sb, pk);
          // ---- the same weights, the rescale factor and the running sum to the partner ----
          const bool pfree =
              __all_sync(0xffffffffu, jj == 0 || mbar_wait_cluster(xp_free, (jj - 1) & 1, wc));
          if (pfree) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              st_async_v4(xp_r + xp_offset(m, 4 * qt + k),
                          make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]),
                          xp_full_r);
            if (qt == 0)
              st_async_v2(xp_r + xp_scalars(m),
                          make_uint2(__float_as_uint(alpha), __float_as_uint(lt)), xp_full_r);
          }
          if (tr) MLA_PTRACE(6, jj);
          // cache rows past the context may hold anything (even NaN): zero their latent half
          // so that 0-weight x garbage cannot reach O
          if (tile_pos0 + kDecodeTok > L) {
            const int tid = sp * 32 + lane;      // 0..127
            const int tok = tid & (kDecodeTok - 1);
            if (tile_pos0 + tok >= L) {
              uint8_t* sbase = slots + slot * lay.slot_bytes;
              for (int k = tid >> 6; k < lb; k += 2) {
                uint4* rowp = reinterpret_cast<uint4*>(sbase + k * kBlk + tok * 128);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) rowp[ch] = make_uint4(0, 0, 0, 0);
              }
            }
          }
          // P (and any O rescale and zeroed rows) complete: hand the tile to the PV issuer
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[sb]);
        }
        // ---- epilogue of this piece: O and lse of the own rows ----
        bool aborted = false;
        write_o(w, tb, te, jj - 1, lt, &aborted);
        if (row_ok && qt == 0) {
          const float lse = (lt > 0.0f && !aborted) ? (mref + __log2f(lt)) * kLn2 : -INFINITY;
          const bool whole = (tb == w.s) && (te == w.s + w.tiles);
          if (whole) p.lse[int64_t(w.b) * p.qH + row] = lse;
          else p.part_lse[int64_t(piece_slot(vc, w.s, per, p.col_groups, cg)) * kPairRows + n] = lse;
        }
        w.s += w.tiles;
        ++w.b;
        if (w.s >= r1) break;
        w.load(p, cg);
      }
    } else if (role == 1) {
      // ------------- sender: the partner's 16 rows of sub-partition sp, partial scores ----
      load_q(sched[0]);
      UnitWalk w{sched[0], sched[1]};
      int jj = 0;
      for (; w.s < r1; w.s += w.tiles, ++w.b) {
        w.load(p, cg);
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        for (int t = tb; t < te; ++t, ++jj) {
          const int sb = jj & 1;
          float x[kHalfTok];
          const bool got = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (jj >> 1) & 1, wc));
          tc_fence_after();
          if (got) {
            tm_ld_x32_s32(trow + kColS + 64 * sb, x);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < kHalfTok; ++c) x[c] = 0.0f;
          }
          if (tr) MLA_PTRACE(3, jj);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[sb]);
          if (t == te - 1 && w.s + w.tiles < r1) load_q(w.b + 1);
          uint32_t pw[kPackWords];
#pragma unroll
          for (int g = 0; g < kHalfTok / 4; ++g) pack_f24(x + 4 * g, pw + 3 * g);
          // into the partner's buffer sb once its owners consumed tile jj - 2 from it: stores
          // from registers over the SM-to-SM network, completing on the partner's mbarrier.
          // The partner's owner thread of this (row, half) is the same lane of its warp sp.
          const bool free_ok = __all_sync(
              0xffffffffu, jj < 2 || mbar_wait_cluster(&xs_free[sb], ((jj - 2) >> 1) & 1, wc));
          if (free_ok) {
            const uint32_t dst = xs_r + sb * kXsBytes;
            const uint32_t rb = sb ? xs_full_r1 : xs_full_r0;
#pragma unroll
            for (int c = 0; c < kPackWords / 4; ++c)
              st_async_v4(dst + xs_offset(sp, lane, c),
                          make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]), rb);
          }
          if (tr) MLA_PTRACE(4, jj);
        }
      }
    } else {
      // ------------- receiver: the partner's weights for its 16 rows of sub-partition sp --
      UnitWalk w{sched[0], sched[1]};
      w.load(p, cg);
      int jj = 0;
      while (true) {
        const int tb = max(w.s, r0), te = min(w.s + w.tiles, r1);
        float lt = 0.0f;
        for (int t = tb; t < te; ++t, ++jj) {
          const int sb = jj & 1;
          const bool rcv = __all_sync(0xffffffffu, mbar_wait_cluster(xp_full, jj & 1, wc));
          if (tr) MLA_PTRACE(7, jj);
          uint32_t pk[kHalfTok / 2];
          float alpha = 1.0f;
          if (rcv) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint4 v = ld_shared_v4(xp_s + xp_offset(m, 4 * qt + k));
              pk[4 * k] = v.x; pk[4 * k + 1] = v.y; pk[4 * k + 2] = v.z; pk[4 * k + 3] = v.w;
            }
            const uint2 sv = ld_shared_v2(xp_s + xp_scalars(m));
            alpha = __uint_as_float(sv.x);
            lt = __uint_as_float(sv.y);
          } else {
#pragma unroll
            for (int c = 0; c < kHalfTok / 2; ++c) pk[c] = 0u;
            lt = 0.0f;
          }
          __syncwarp();
          // consumed into registers: release the buffer (relaxed) and re-arm it for tile jj + 1
          if (lane == 1) mbar_arrive_remote_relaxed(xp_free_r);
          if (sp == 0 && lane == 0 && rcv) mbar_arrive_expect_tx_relaxed(xp_full, kXpBytes);
          // the owner moved its reference: rescale these rows of this CTA's O half the same way
          if (t > tb && __any_sync(0xffffffffu, alpha != 1.0f)) rescale_o(jj, alpha);
          if (jj >= 2) {
            __all_sync(0xffffffffu, mbar_wait(&pv_done[sb], ((jj - 2) >> 1) & 1, wc));
            tc_fence_after();
          }
          tm_st_x16_s16(trow + kColP + 32 * sb, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[sb]);
          if (tr) MLA_PTRACE(11, jj);
        }
        // ---- epilogue of this piece: O of the partner's rows (this CTA's latent half) ----
        bool aborted = false;
        write_o(w, tb, te, jj - 1, lt, &aborted);
        w.s += w.tiles;
        ++w.b;
        if (w.s >= r1) break;
        w.load(p, cg);
      }
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
  return launch_pdl(mla_decode_pair_kernel, grid, dim3(kThreads), smem, stream, 2, p);
}

}  // namespace mla
