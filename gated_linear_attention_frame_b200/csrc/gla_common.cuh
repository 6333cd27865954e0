// gla_common.cuh -- shapes, shared-memory tile geometry and the split of the
// token tiles across CTAs, shared by the three kernels and the host code.
#pragma once

#include <cstdint>

namespace gla {

constexpr int kTileTokens = 128;  // tokens per tile (MMA M for the output, K for the increment)

// Swizzled tile geometry for head dim D.  Tiles are kept in the canonical
// tcgen05 shared-memory layout: rows of kRowBytes (128-byte swizzle for D >=
// 64, 64-byte swizzle for D = 32), grouped in atoms of kAtomElems columns.
template <int D>
struct Geo {
  static_assert(D == 32 || D == 64 || D == 128, "head dim must be 32, 64 or 128");
  static constexpr int kAtomElems = (D >= 64) ? 64 : 32;         // bf16 per swizzle row
  static constexpr int kRowBytes = kAtomElems * 2;                // 128 or 64
  static constexpr int kAtoms = D / kAtomElems;                   // atoms across the head dim
  static constexpr int kGroupBytes = 8 * kRowBytes;               // 8-row core-matrix group
  static constexpr uint32_t kLayout = (D >= 64) ? 2u : 4u;        // SW128 / SW64 descriptor code
  static constexpr int kAtomTileBytes = kTileTokens * kRowBytes;  // one atom of a 128-token tile
  static constexpr int kTileBytes = kTileTokens * D * 2;          // a [128 x D] bf16 tile
  static constexpr int kChunksPerRow = D / 8;                     // 16-byte chunks per token row
  // Increment (state) rows: D value columns plus the normaliser column.
  static constexpr int kStateRows = D + 1;
  // Output-kernel B operand: state rows padded to a multiple of 16 (MMA N).
  static constexpr int kNPad = D + 16;
  // One frame's prefix state S_f^T in bf16 as written by the scan for the
  // output kernel: kAtoms blocks of kStateRows swizzled rows.
  static constexpr int kImageAtomBytes = kStateRows * kRowBytes;
  static constexpr int kImageBytes = kAtoms * kImageAtomBytes;
  // fp32 partial increment [kStateRows][D] (row D = normaliser column).
  static constexpr int kPartialFloats = kStateRows * D;

  // Physical 16-byte chunk slot of logical chunk `c` (within an atom) of
  // swizzled row `r`.
  __host__ __device__ static constexpr int swz(int r, int c) {
    return (D >= 64) ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
  }
};

// Contiguous split of W token tiles over G CTAs: CTA c owns tiles
// [lo(c), lo(c+1)) with lo(c) = floor(c * W / G).
struct TileSplit {
  int64_t W;  // tiles
  int32_t G;  // CTAs
  __host__ __device__ int64_t lo(int64_t c) const { return (c * W) / G; }
  // CTA owning tile x: the largest c with lo(c) <= x.
  __host__ __device__ int64_t owner(int64_t x) const { return ((x + 1) * G - 1) / W; }
};

// Assignment of the token tiles of all units to the G persistent CTAs of the
// increment and output kernels.  Unit u = (b * F + f) * H + h is one (batch,
// frame, head); it has tpu = ceil(T / 128) tiles.
//
//  * Full rounds: while at least G units remain, round r gives unit r*G + c
//    to CTA c whole.  Consecutive CTAs then hold consecutive heads of the same
//    frame and move through the same token tiles at the same pace, so the
//    CTAs of one frame read and write whole token rows (all heads) of q, k, v
//    and out together: DRAM pages are opened once, not once per head.
//  * Tail: the remaining units' tiles (fewer than G units) are split
//    contiguously (TileSplit) over min(G, tail tiles) CTAs, so that every
//    CTA of the tail owns at least one tile.
//
// The increment kernel writes one fp32 partial per (unit, CTA) segment, at
// slot u for a full-round unit and at slot u + c for a tail unit (unique:
// along the tail, u and c never decrease and one of them grows at every new
// segment).  Slots < units + G.
struct WorkPlan {
  int32_t units;     // B * F * H
  int32_t tpu;       // tiles per unit
  int32_t G;         // CTAs
  int32_t rounds;    // full rounds = units / G
  int64_t tail_W;    // tiles in the tail = (units - rounds * G) * tpu

  __host__ __device__ static WorkPlan make(int64_t units, int tpu, int G) {
    WorkPlan w;
    w.units = static_cast<int32_t>(units);
    w.tpu = tpu;
    w.G = G;
    w.rounds = static_cast<int32_t>(units / G);
    w.tail_W = (units - static_cast<int64_t>(w.rounds) * G) * tpu;
    return w;
  }
  __host__ __device__ int32_t full_units() const { return rounds * G; }
  __host__ __device__ int32_t tail_G() const {
    return tail_W < G ? static_cast<int32_t>(tail_W) : G;
  }
  __host__ __device__ TileSplit tail() const { return TileSplit{tail_W, tail_G()}; }
  // First and last CTA holding a partial of unit u (slots u + first .. u + last;
  // a full-round unit has exactly one partial, at slot u).
  __host__ __device__ void slot_range(int64_t u, int32_t& first, int32_t& last) const {
    if (u < full_units()) {
      first = last = 0;
      return;
    }
    const int64_t x0 = (u - full_units()) * tpu;
    first = static_cast<int32_t>(tail().owner(x0));
    last = static_cast<int32_t>(tail().owner(x0 + tpu - 1));
  }
  __host__ __device__ int64_t slot(int64_t u, int32_t cta) const {
    return u < full_units() ? u : u + cta;
  }
};

// Walks the tiles of one CTA in order: its full-round units, then its tail
// range.  `first` / `last` mark the first / last tile of a segment (a run of
// tiles of one unit inside this CTA).  All arithmetic is incremental.
struct TileCursor {
  int32_t u;      // unit of the current tile
  int32_t t;      // tile index within the unit
  bool first, last;
  int64_t i;      // position in this CTA's sequence
  int64_t n;      // tiles of this CTA
  int64_t n_full; // tiles of this CTA in full rounds
  int64_t x_lo;   // first tail tile of this CTA
  int32_t tpu, G, cta, U_full;

  __host__ __device__ void init(const WorkPlan& wp, int32_t c) {
    tpu = wp.tpu;
    G = wp.G;
    cta = c;
    U_full = wp.full_units();
    n_full = static_cast<int64_t>(wp.rounds) * tpu;
    const TileSplit ts = wp.tail();
    const bool in_tail = c < wp.tail_G();
    x_lo = in_tail ? ts.lo(c) : 0;
    const int64_t x_hi = in_tail ? ts.lo(c + 1) : 0;
    n = n_full + (x_hi - x_lo);
    i = 0;
    if (n_full > 0) {
      u = c;
      t = 0;
    } else {
      enter_tail();
    }
    flags();
  }
  __host__ __device__ bool valid() const { return i < n; }
  __host__ __device__ void enter_tail() {
    u = U_full + static_cast<int32_t>(x_lo / tpu);
    t = static_cast<int32_t>(x_lo % tpu);
  }
  __host__ __device__ void flags() {
    first = (i == 0) || (t == 0) || (i == n_full);
    last = (i == n - 1) || (t == tpu - 1) || (i == n_full - 1);
  }
  __host__ __device__ void advance() {
    ++i;
    if (i == n_full) {
      enter_tail();
    } else if (++t == tpu) {
      t = 0;
      u += (i < n_full) ? G : 1;
    }
    flags();
  }
  __host__ __device__ int64_t slot() const { return u < U_full ? int64_t(u) : int64_t(u) + cta; }
};

}  // namespace gla
