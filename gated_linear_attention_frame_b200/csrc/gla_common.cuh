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
  int64_t W;  // total tiles = units * tiles_per_unit
  int32_t G;  // CTAs
  __host__ __device__ int64_t lo(int64_t c) const { return (c * W) / G; }
  // CTA owning tile x: the largest c with lo(c) <= x.
  __host__ __device__ int64_t owner(int64_t x) const { return ((x + 1) * G - 1) / W; }
};

// Unit u = (b * F + f) * H + h indexes one (batch, frame, head).  A unit's
// increment is summed from the partials of every CTA that owns one of its
// tiles; the partial of (unit u, CTA c) lives at slot u + c, which is unique
// because both u and c only grow along the tile order.

}  // namespace gla
