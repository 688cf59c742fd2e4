// decode_sched.cuh - the work schedule shared by the decode kernels.
//
// A "unit" is (sequence b, block cg of query rows); its work is ceil(L_b / 64) page tiles
// (one tile when L_b is 0). The units of one row block are laid end to end and cut into
// `vgrid` equal ranges, one per virtual CTA (a CTA, or a cluster working as one), so
// ragged lengths balance. A unit a virtual CTA holds whole is written straight to the
// outputs; a unit cut between virtual CTAs leaves one partial (o, lse) per piece, merged
// afterwards with the log-sum-exp identity.
#pragma once

#include "kernels.h"
#include "ptx.cuh"

namespace mla {

MLA_DEVICE int unit_tiles(int L) { return L > 0 ? (L + kDecodeTok - 1) / kDecodeTok : 1; }

// Context length of sequence b if it is within the bounds the launch was planned for,
// else 0 (the unit then produces zeros and lse = -inf, and the error word is set).
MLA_DEVICE int valid_len(const DecodeParams& p, int L) {
  const bool ok = L >= p.q_len && L <= p.max_seq_len &&
                  int64_t(L) <= int64_t(p.max_pages) * kDecodeTok;
  return ok ? L : 0;
}

// Position of tile number j in a ring of n cache slots, kept incrementally: slot = j % n
// and round = j / n without a division on the issue paths (an integer division by a
// runtime value there measurably lengthens the per-tile loop).
struct SlotRing {
  int n, slot, round;
  MLA_DEVICE explicit SlotRing(int nslot) : n(nslot), slot(0), round(0) {}
  MLA_DEVICE void next() {
    if (++slot == n) {
      slot = 0;
      ++round;
    }
  }
};

// The walk over the sequences a range touches; every role runs the same walk.
struct UnitWalk {
  int b, s;       // sequence and the index of its first tile in this row block's tile space
  int tiles, L, u;
  MLA_DEVICE void load(const DecodeParams& p, int cg) {
    L = valid_len(p, p.seq_lens[b]);
    tiles = unit_tiles(L);
    u = b * p.col_groups + cg;
  }
};

// Partial-result slot of virtual CTA i (of row block cg) holding a piece of a unit whose
// first tile is s, when ranges are `per` tiles long: slot 0 holds a range's first piece,
// slot 1 its last. A unit is the first piece of every range it reaches except possibly the
// one where it starts.
MLA_DEVICE int piece_slot(int i, int s, int per, int col_groups, int cg) {
  const int i0 = s / per;
  return 2 * (i * col_groups + cg) + ((i == i0 && s != i0 * per) ? 1 : 0);
}

// Tile range [r0, r1) of virtual CTA vc among vgrid, and the sequence holding tile r0.
// All NT threads of the CTA call it. Writes sched[0] = that sequence (-1 if none),
// sched[1] = its first tile, sched[2] = r0, sched[3] = r1, sched[4] = range length;
// sched[5] and warp_sum[NT / 32] are scratch. Lengths outside the planned bounds are
// reported (MLA_DEVERR_BOUNDS) when report_bounds is set.
template <int NT>
MLA_DEVICE void find_tile_range(const DecodeParams& p, int vc, int vgrid, bool report_bounds,
                                int* warp_sum, int* sched) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int total = 0;
  for (int b = threadIdx.x; b < p.batch; b += NT) {
    const int Lv = valid_len(p, p.seq_lens[b]);
    if (Lv == 0 && report_bounds && p.dev_error) atomicOr(p.dev_error, MLA_DEVERR_BOUNDS);
    total += unit_tiles(Lv);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  if (lane == 0) warp_sum[warp] = total;
  __syncthreads();
  total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) total += warp_sum[w];
  const int per = max(1, (total + vgrid - 1) / vgrid);
  const int r0 = min(total, vc * per);
  const int r1 = min(total, r0 + per);
  __syncthreads();
  if (threadIdx.x == 0) {
    sched[0] = -1;
    sched[2] = r0;
    sched[3] = r1;
    sched[4] = per;
    sched[5] = 0;   // running tile count before the current chunk of sequences
  }
  __syncthreads();
  // chunked exclusive scan over the sequences until the one holding tile r0 is found
  for (int b0 = 0; b0 < p.batch && r0 < r1; b0 += NT) {
    const int b = b0 + threadIdx.x;
    const int t = b < p.batch ? unit_tiles(valid_len(p, p.seq_lens[b])) : 0;
    int incl = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int before = sched[5];
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    const int start = before + incl - t;
    if (b < p.batch && start <= r0 && r0 < start + t) {
      sched[0] = b;
      sched[1] = start;
    }
    __syncthreads();
    if (threadIdx.x == NT - 1) sched[5] = before + incl;
    __syncthreads();
    if (sched[0] >= 0) break;
  }
}

}  // namespace mla
