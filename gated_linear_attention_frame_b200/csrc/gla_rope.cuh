// gla_rope.cuh -- 3D rotary position embedding for the gated linear attention
// kernels (the SANA-Video talk's "3D RoPE for the linear attention", temporal
// modelling segment; the formula is this library's reading, RoFormer form):
//
//   token t of frame f sits at (p_t, p_y, p_x) = (frame_offset + f, t / grid_w, t % grid_w);
//   the head dim is split into blocks [temporal d_t | height d_y | width d_x],
//   each a multiple of 8; pair j of a block of n features (features 2j, 2j+1
//   of the block) turns by p_axis * theta^(-2j/n).
//   The numerator uses the rotated feature maps R_t phi(q_t), R_t phi(k_t);
//   the normaliser keeps the un-rotated phi(q_t) . sum phi(k).
//
// Since every block is a multiple of 8 features, each 16-byte chunk of a
// token row (8 bf16, 4 pairs) belongs to one block.  A thread owns chunk c of
// the rows r0, r0 + P, r0 + 2P, ... of a tile (P = rows per pass of the ReLU
// warps).  It reads the (cos, sin) of its 4 pairs for its first row from a
// small fp32 table and steps to the next rows by angle addition: from one row
// to the next the column advances by P mod grid_w or by that minus grid_w
// (wrapping to the next latent row), and the row index by floor(P / grid_w)
// or one more; the (cos, sin) of both increments of every pair are in the
// table too.  Table (built once per call by gla_rope_table_kernel in fp64,
// rounded to fp32):
//   section t: [frames][d_t / 2]   (positions frame_offset .. frame_offset + F - 1)
//   section y: [rows][d_y / 2]     (rows = ceil(T / grid_w))
//   section x: [cols][d_x / 2]     (cols = min(T, grid_w))
//   section inc: [2][d / 2]        (per pair: the no-wrap and the wrap increment;
//                                   (1, 0) for the temporal block)
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace gla {

struct RopeGeo {
  const float4* table;  // (cos_j, sin_j, cos_j+1, sin_j+1) pairs; see above
  int dt, dy, dx;       // feature blocks (multiples of 8, dt + dy + dx = d)
  int grid_w;           // tokens per latent row
  int rows, cols;       // positions of the height and width sections
  int frames;           // positions of the temporal section
  int frame_offset;
  int64_t sec_y, sec_x; // start of the height / width sections, in (cos, sin) pairs
  int64_t sec_inc;      // start of the increment section
  int rpp;              // token rows between a thread's consecutive rows
};

// The block of chunk c (features 8c .. 8c+7) and where its pairs sit.
struct RopeChunk {
  int blk;      // 0 temporal, 1 height, 2 width
  int npairs;   // pairs per position in the block's section
  int j0;       // first pair of the chunk within the block
  int64_t sec;  // start of the block's section
};

__device__ __forceinline__ RopeChunk rope_chunk(const RopeGeo& g, int c) {
  const int e = 8 * c;
  if (e < g.dt) return RopeChunk{0, g.dt / 2, e / 2, 0};
  if (e < g.dt + g.dy) return RopeChunk{1, g.dy / 2, (e - g.dt) / 2, g.sec_y};
  return RopeChunk{2, g.dx / 2, (e - g.dt - g.dy) / 2, g.sec_x};
}

// Rotate the 4 pairs of one chunk (packed bf16) by the angles whose
// (cos, sin) are in cs01 (pairs 0, 1) and cs23 (pairs 2, 3); rounds to bf16.
__device__ __forceinline__ uint32_t rotate_pair(uint32_t w, float c, float s) {
  const float x0 = bf16lo_to_f32(w), x1 = bf16hi_to_f32(w);
  return pack_bf16x2(fmaf(x0, c, -x1 * s), fmaf(x0, s, x1 * c));
}

__device__ __forceinline__ void rotate8(uint4& w, const float4& cs01, const float4& cs23) {
  w.x = rotate_pair(w.x, cs01.x, cs01.y);
  w.y = rotate_pair(w.y, cs01.z, cs01.w);
  w.z = rotate_pair(w.z, cs23.x, cs23.y);
  w.w = rotate_pair(w.w, cs23.z, cs23.w);
}

// Tracks the position of one thread's token rows r0, r0 + step, ... of a
// tile along its chunk's axis; `next` moves to the next row.
struct RopeRowPos {
  int tok, y, x;
  __device__ __forceinline__ void start(int tok0, int grid_w) {
    tok = tok0;
    y = tok0 / grid_w;
    x = tok0 - y * grid_w;
  }
  __device__ __forceinline__ void next(int step, int grid_w) {
    tok += step;
    x += step;
    while (x >= grid_w) {
      x -= grid_w;
      ++y;
    }
  }
};

// The chunk's (cos, sin) entries for the current row; rows past the frame's
// end (zero data) use position 0.
__device__ __forceinline__ void rope_coeffs(const RopeGeo& g, const RopeChunk& rc, int frame,
                                            const RopeRowPos& rp, int T, float4& cs01,
                                            float4& cs23) {
  int pos = rc.blk == 0 ? frame : (rc.blk == 1 ? rp.y : rp.x);
  if (rp.tok >= T) pos = 0;
  const int64_t idx = (rc.sec + static_cast<int64_t>(pos) * rc.npairs + rc.j0) >> 1;
  cs01 = __ldg(g.table + idx);
  cs23 = __ldg(g.table + idx + 1);
}

// (cos, sin) of a thread's 4 pairs on its current row, and the two
// increments that lead to its next row.
struct RopeStep {
  float4 cs01, cs23;  // current row
  float4 ia01, ia23;  // next row on the same latent row (no wrap)
  float4 ib01, ib23;  // next row after a wrap
  int step_mod;       // rpp mod grid_w
  bool moving;        // false for the temporal block (one angle per frame)
};

// Once per thread: the increments of chunk c (pairs 4c .. 4c+3).
__device__ __forceinline__ void rope_step_init(const RopeGeo& g, int c, int half_d, RopeStep& st) {
  const int64_t ia = (g.sec_inc + 4 * c) >> 1;
  const int64_t ib = (g.sec_inc + half_d + 4 * c) >> 1;
  st.ia01 = __ldg(g.table + ia);
  st.ia23 = __ldg(g.table + ia + 1);
  st.ib01 = __ldg(g.table + ib);
  st.ib23 = __ldg(g.table + ib + 1);
  st.step_mod = g.rpp % g.grid_w;
  st.moving = 8 * c >= g.dt;
}

__device__ __forceinline__ float4 cmul2(const float4& a, const float4& b) {
  return make_float4(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x, a.z * b.z - a.w * b.w,
                     a.z * b.w + a.w * b.z);
}

// Move to the next row (rp still describes the current row).
__device__ __forceinline__ void rope_step_next(RopeStep& st, const RopeRowPos& rp, int grid_w) {
  if (!st.moving) return;
  const bool wrap = rp.x + st.step_mod >= grid_w;
  st.cs01 = cmul2(st.cs01, wrap ? st.ib01 : st.ia01);
  st.cs23 = cmul2(st.cs23, wrap ? st.ib23 : st.ia23);
}

// One thread per (cos, sin) entry of the three sections, in fp64.
__global__ void __launch_bounds__(256) gla_rope_table_kernel(float2* table, RopeGeo g,
                                                             double log2_theta) {
  const int64_t nt = static_cast<int64_t>(g.frames) * (g.dt / 2);
  const int64_t ny = static_cast<int64_t>(g.rows) * (g.dy / 2);
  const int64_t nx = static_cast<int64_t>(g.cols) * (g.dx / 2);
  const int half_d = (g.dt + g.dy + g.dx) / 2;
  const int64_t total = nt + ny + nx + 2 * half_d;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t k = i;
    int n, pos, j;
    if (k >= nt + ny + nx) {
      // increments: which = 0 (no wrap) or 1 (wrap), pair pp of the head dim
      k -= nt + ny + nx;
      const int which = static_cast<int>(k / half_d);
      const int pp = static_cast<int>(k % half_d);
      const int step_mod = g.rpp % g.grid_w, step_div = g.rpp / g.grid_w;
      int delta = 0;
      if (2 * pp < g.dt) {
        n = g.dt;
        j = pp;
      } else if (2 * pp < g.dt + g.dy) {
        n = g.dy;
        j = pp - g.dt / 2;
        delta = step_div + which;
      } else {
        n = g.dx;
        j = pp - (g.dt + g.dy) / 2;
        delta = which ? step_mod - g.grid_w : step_mod;
      }
      const double freq = exp2(-2.0 * j / n * log2_theta);
      double s, c;
      sincos(static_cast<double>(delta) * freq, &s, &c);
      table[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
      continue;
    }
    if (k < nt) {
      n = g.dt;
      pos = g.frame_offset + static_cast<int>(k / (n / 2));
      j = static_cast<int>(k % (n / 2));
    } else if ((k -= nt) < ny) {
      n = g.dy;
      pos = static_cast<int>(k / (n / 2));
      j = static_cast<int>(k % (n / 2));
    } else {
      k -= ny;
      n = g.dx;
      pos = static_cast<int>(k / (n / 2));
      j = static_cast<int>(k % (n / 2));
    }
    const double freq = exp2(-2.0 * j / n * log2_theta);
    double s, c;
    sincos(static_cast<double>(pos) * freq, &s, &c);
    table[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

}  // namespace gla
