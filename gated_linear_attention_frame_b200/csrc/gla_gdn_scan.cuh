// gla_gdn_scan.cuh -- the frame-wise gated delta-rule scan.
//
// The SANA-WM pages describe frame-wise Gated DeltaNet: the recurrent state of
// the linear attention gets decay gates and delta-rule corrections.  This
// library reads it as (per (b, h), frames in order, a_f = sigmoid(g),
// beta_f = sigmoid(beta logit), K~ = relu(K_f), M_f = K~^T K~, dS_f = K~^T [V_f | 1]):
//   S_f = a_f S_{f-1} + beta_f K~^T ([V_f | 1] - a_f K~ S_{f-1})
//       = a_f (S_{f-1} - beta_f M_f S_{f-1}) + beta_f dS_f
// The frame's keys read what the decayed state holds for them and write back
// only the difference.  Unlike the plain gated scan, the update couples the
// d rows of S through M_f, but every state column j is still independent:
//   S_f[:, j] = a_f (S_{f-1}[:, j] - beta_f M_f S_{f-1}[:, j]) + beta_f dS_f[:, j].
// Two kernels run this recurrence: gla_gdn_scan_tc_kernel (d = 128, the
// product on tcgen05, described with it below) and gla_gdn_scan_kernel
// (d = 32, 64, CUDA cores), described here.
// One block owns a group of columns of one (b, h) and loops over the frames:
// a producer warp bulk-copies M_f (fp32, d x d, the increment kernel's Gram
// partial) into a two-stage shared-memory ring; eight consumer warps each own
// d/8 rows of S and every lane one or two of the group's columns, so a warp
// reads each row k of M_f once (a broadcast) for all its columns and forms
// M_f S_{f-1}[:, j] in fp32 from the previous state held in shared memory
// (row-major [i][j], columns contiguous).  Each lane then adds the frame's
// dS_f rows (read from global memory before the contraction, so the loads
// overlap it), writes the next state to the other buffer and the bf16 S_f^T
// image that the output kernel reads.  Further partials of a unit that the
// tile schedule split over several increment CTAs: gla_gram_reduce_kernel
// first adds their Gram partials into the unit's first slot (the scan then
// reads one M_f per frame); their dS rows are summed by the scan from global
// memory.  The warps pass a frame to each other through an mbarrier, so every
// wait is bounded.
#pragma once

#include <type_traits>

#include "gla_common.cuh"
#include "gla_increment.cuh"
#include "gla_scan.cuh"  // add8
#include "sm100_ptx.cuh"

namespace gla {

struct GdnScanParams {
  const float* partial;   // dS_f partials [slots][d + 1][d] (transposed, row d = normaliser)
  const float* mpartial;  // M_f partials [slots][d][d] (d = 128: a whole unit's GramImage pair)
  const uint8_t* mtail;   // d = 128: GramImage pairs of the tail units [tail units][d * d * 4 B]
  const float* gate;      // [B, F, H] decay logits
  const float* beta;      // [B, F, H] write-strength logits
  const float* state_in;  // [B, H, d, d + 1] or nullptr
  float* state_out;       // [B, H, d, d + 1] or nullptr
  uint8_t* image;         // [units][kImageBytes] or nullptr
  WorkPlan wp;
  int H, F, tpu;
  int groups;             // blocks per (b, h)
  int cols;               // state columns per block (the last block may have fewer)
};

template <int D>
struct GdnScanCfg {
  static constexpr int kConsumerWarps = (D / 8 < 8) ? D / 8 : 8;  // each warp >= 8 rows
  static constexpr int kConsumers = 32 * kConsumerWarps;
  static constexpr int kThreads = kConsumers + 32;
  static constexpr int kRowsPerWarp = D / kConsumerWarps;  // 16 at d = 128, else 8
  static constexpr int kMaxCols = 44;                      // >= ceil((D + 1) / 3); <= 64
  static_assert(3 * kMaxCols >= D + 1 && kMaxCols <= 64, "columns per block");
  static constexpr int kColStride = kMaxCols;              // state tile row stride (floats)
  static constexpr int kMBytes = D * D * 4;
  static constexpr int kStageBytes = kMBytes + 16;
  static constexpr int kStages = 2;
  static constexpr int kTileBytes = D * kColStride * 4;    // one state buffer [D][cols]
  static constexpr int kBarCount = 2 * kStages + 1;
  static constexpr int kSmemBytes = 128 + kStages * kStageBytes + 2 * kTileBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
};

struct GdnStageHeader {
  int32_t c0, c1;  // the unit's partial slots u + c0 .. u + c1
  float a, beta;
};

template <int D>
__global__ void __launch_bounds__(GdnScanCfg<D>::kThreads, 1)
    gla_gdn_scan_kernel(const GdnScanParams p) {
  using G = Geo<D>;
  using C = GdnScanCfg<D>;
  constexpr int PF = IncCfg<D>::kPartialFloats;
  constexpr int S = C::kStages;
  constexpr int RPW = C::kRowsPerWarp;
  constexpr int CS = C::kColStride;
  constexpr unsigned kCode = 64u;
  constexpr int kCW = C::kConsumerWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  auto stage = [&](int s) { return smem + s * C::kStageBytes; };  // [M | hdr]
  float* sbuf0 = reinterpret_cast<float*>(smem + S * C::kStageBytes);
  float* sbuf1 = sbuf0 + D * CS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + 2 * C::kTileBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t fdone = bar0 + 8u * (2 * S);  // every consumer warp finished a frame
  volatile int* abort = reinterpret_cast<volatile int*>(bars + C::kBarCount);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.groups;
  const int grp = blockIdx.x % p.groups;
  const int j0 = grp * p.cols;
  const int ncols = (D + 1 - j0 < p.cols) ? D + 1 - j0 : p.cols;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t u0 = static_cast<int64_t>(b) * p.F * p.H + h;
  const int64_t srow = static_cast<int64_t>(bh) * D * (D + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kCW);
    }
    mbar_init(fdone, kCW);
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const bool stream = p.tpu > 0 && p.F > 0;
  if (warp == kCW) {
    // ---------------------------------------------------------------- producer
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the increment kernel
    if (stream) {
      float gl = 0.f, bl = 0.f;
      int f = 0;
      for (; f < p.F; ++f) {
        if ((f & 31) == 0) {
          const int ff = f + lane;
          gl = ff < p.F ? __ldg(p.gate + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
          bl = ff < p.F ? __ldg(p.beta + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
        }
        const float g = __shfl_sync(0xffffffffu, gl, f & 31);
        const float bb = __shfl_sync(0xffffffffu, bl, f & 31);
        int ok = 1;
        if (lane == 0) {
          const int s = f % S;
          ok = mbar_wait(empty(s), static_cast<uint32_t>(((f / S) & 1) ^ 1), abort, kCode) ? 1 : 0;
          if (ok) {
            const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
            int32_t c0, c1;
            p.wp.slot_range(u, c0, c1);
            GdnStageHeader* hdr = reinterpret_cast<GdnStageHeader*>(stage(s) + C::kMBytes);
            hdr->c0 = c0;
            hdr->c1 = c1;
            hdr->a = 1.0f / (1.0f + expf(-g));
            hdr->beta = 1.0f / (1.0f + expf(-bb));
            mbar_arrive_expect_tx(full(s), C::kMBytes);
            bulk_load(smem_u32(stage(s)), p.mpartial + (u + c0) * static_cast<int64_t>(D) * D,
                      C::kMBytes, full(s));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (lane == 0)
        for (int k = (f > S ? f - S : 0); k < f; ++k)
          mbar_wait_drain(full(k % S), static_cast<uint32_t>((k / S) & 1));
    }
  } else {
    // --------------------------------------------------------------- consumers
    float* sprev = sbuf0;
    float* snext = sbuf1;
    // state_in columns j0 .. j0+ncols-1 -> sprev[i][jl]
    for (int idx = threadIdx.x; idx < D * ncols; idx += C::kConsumers) {
      const int jl = idx % ncols, i = idx / ncols;
      sprev[i * CS + jl] =
          p.state_in != nullptr ? p.state_in[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jl]
                                : 0.f;
    }
    named_bar_sync(1, C::kConsumers);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int CPA = G::kAtomElems / 8;
    const int i0 = warp * RPW;             // this warp's rows
    const bool has0 = lane < ncols;        // column lane
    const bool has1 = lane + 32 < ncols;   // column lane + 32
    for (int f = 0; f < p.F; ++f) {
      const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
      float a, beta;
      int32_t c0 = 0, c1 = 0;
      const float* mst = nullptr;
      if (stream) {
        const int s = f % S;
        if (!warp_wait(full(s), static_cast<uint32_t>((f / S) & 1), abort, kCode)) break;
        const GdnStageHeader hd = *reinterpret_cast<const GdnStageHeader*>(stage(s) + C::kMBytes);
        a = hd.a;
        beta = hd.beta;
        c0 = hd.c0;
        c1 = hd.c1;
        mst = reinterpret_cast<const float*>(stage(s));
      } else {
        // frames without tokens: no write, the state only decays
        a = 1.0f / (1.0f + expf(-__ldg(p.gate + u)));
        beta = 0.f;
      }
      float acc0[RPW], acc1[RPW], ds0[RPW], ds1[RPW];
#pragma unroll
      for (int r = 0; r < RPW; ++r) acc0[r] = acc1[r] = ds0[r] = ds1[r] = 0.f;
      if (stream) {
        // dS_f rows of this lane's columns, issued before the contraction
        for (int cc = c0; cc <= c1; ++cc) {
          const float* base = p.partial + (u + cc) * PF + i0;
          if (has0) {
            const float4* x = reinterpret_cast<const float4*>(base + static_cast<int64_t>(j0 + lane) * D);
#pragma unroll
            for (int r4 = 0; r4 < RPW / 4; ++r4) {
              const float4 v4 = __ldg(x + r4);
              ds0[4 * r4] += v4.x; ds0[4 * r4 + 1] += v4.y; ds0[4 * r4 + 2] += v4.z; ds0[4 * r4 + 3] += v4.w;
            }
          }
          if (has1) {
            const float4* x =
                reinterpret_cast<const float4*>(base + static_cast<int64_t>(j0 + lane + 32) * D);
#pragma unroll
            for (int r4 = 0; r4 < RPW / 4; ++r4) {
              const float4 v4 = __ldg(x + r4);
              ds1[4 * r4] += v4.x; ds1[4 * r4 + 1] += v4.y; ds1[4 * r4 + 2] += v4.z; ds1[4 * r4 + 3] += v4.w;
            }
          }
        }
        // (M_f S_{f-1})[i0 .. i0+RPW-1, j]; M symmetric: row k of M is column k.
        // The second column of each lane is only formed when the block has one.
        auto contract = [&](const float* mrow, bool from_smem, auto two) {
#pragma unroll 2
          for (int k = 0; k < D; ++k) {
            float m[RPW];
            const float4* mk = reinterpret_cast<const float4*>(mrow + k * D + i0);
#pragma unroll
            for (int r4 = 0; r4 < RPW / 4; ++r4) {
              const float4 v4 = from_smem ? mk[r4] : __ldg(mk + r4);
              m[4 * r4] = v4.x; m[4 * r4 + 1] = v4.y; m[4 * r4 + 2] = v4.z; m[4 * r4 + 3] = v4.w;
            }
            const float s0 = has0 ? sprev[k * CS + lane] : 0.f;
#pragma unroll
            for (int r = 0; r < RPW; ++r) acc0[r] = fmaf(m[r], s0, acc0[r]);
            if constexpr (decltype(two)::value) {
              const float s1 = has1 ? sprev[k * CS + lane + 32] : 0.f;
#pragma unroll
              for (int r = 0; r < RPW; ++r) acc1[r] = fmaf(m[r], s1, acc1[r]);
            }
          }
        };
        // the unit's Gram partials were added into slot c0 beforehand
        if (ncols > 32)
          contract(mst, true, std::true_type{});
        else
          contract(mst, true, std::false_type{});
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(f % S));
      }
      // S_f = a (S_{f-1} - beta M S_{f-1}) + beta dS_f, this lane's columns
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const bool has = half == 0 ? has0 : has1;
        if (!has) continue;
        const int jl = lane + 32 * half;
        float sn[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const float sp = sprev[(i0 + r) * CS + jl];
          const float ac = half == 0 ? acc0[r] : acc1[r];
          const float dd = half == 0 ? ds0[r] : ds1[r];
          sn[r] = a * fmaf(-beta, ac, sp) + beta * dd;
          snext[(i0 + r) * CS + jl] = sn[r];
        }
        if (p.image != nullptr) {
          const int j = j0 + jl;
#pragma unroll
          for (int q8 = 0; q8 < RPW / 8; ++q8) {
            const int ch = i0 / 8 + q8;  // 8-feature chunk of row j of S_f^T
            uint4 w;
            w.x = pack_bf16x2(sn[8 * q8 + 0], sn[8 * q8 + 1]);
            w.y = pack_bf16x2(sn[8 * q8 + 2], sn[8 * q8 + 3]);
            w.z = pack_bf16x2(sn[8 * q8 + 4], sn[8 * q8 + 5]);
            w.w = pack_bf16x2(sn[8 * q8 + 6], sn[8 * q8 + 7]);
            *reinterpret_cast<uint4*>(p.image + u * G::kImageBytes +
                                      (ch / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                                      G::swz(j, ch % CPA) * 16) = w;
          }
        }
      }
      // hand the frame over: every warp must have read sprev and written snext
      __syncwarp();
      if (lane == 0) mbar_arrive(fdone);
      if (!warp_wait(fdone, static_cast<uint32_t>(f & 1), abort, kCode)) break;
      float* t = sprev;
      sprev = snext;
      snext = t;
    }
    if (p.state_out != nullptr) {
      for (int idx = threadIdx.x; idx < D * ncols; idx += C::kConsumers) {
        const int jl = idx % ncols, i = idx / ncols;
        p.state_out[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jl] = sprev[i * CS + jl];
      }
    }
  }
  __syncwarp();
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// For the units that the tile schedule split over several increment CTAs
// (the tail units), add the Gram partials of slots u + c0 + 1 .. u + c1 into
// slot u + c0, so that the scan streams one M_f per frame.  Grid: (tail units,
// column blocks); a fixed summation order.  Launched as a programmatic
// dependent of the increment kernel; the scan depends on it in turn.
template <int D>
__global__ void __launch_bounds__(256) gla_gram_reduce_kernel(float* mpartial, WorkPlan wp) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t u = static_cast<int64_t>(wp.full_units()) + blockIdx.x;
  int32_t c0, c1;
  wp.slot_range(u, c0, c1);
  if (c1 > c0) {
    float4* dst = reinterpret_cast<float4*>(mpartial + (u + c0) * static_cast<int64_t>(D) * D);
    for (int x = blockIdx.y * blockDim.x + threadIdx.x; x < D * D / 4;
         x += gridDim.y * blockDim.x) {
      float4 acc = dst[x];
      for (int cc = c0 + 1; cc <= c1; ++cc) {
        const float4 v =
            reinterpret_cast<const float4*>(mpartial + (u + cc) * static_cast<int64_t>(D) * D)[x];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      dst[x] = acc;
    }
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gla

namespace gla {

// The tail units at d = 128 (tensor-core scan): the Gram partials of slots
// u + c0 .. u + c1 are summed in fp32 (in slot order) and written as the
// unit's GramImage pair into mtail, and the dS partials of those slots are
// summed into slot u + c0, so that the scan streams one M_f image and one
// dS_f per frame.  Grid: (tail units, kGramParts + kDsParts); y < kGramParts
// takes 2 of the 16 K chunks of M_f (one 8-element chunk of one row per
// thread), the rest interleaved float4s of the dS rows.
constexpr int kGramParts = 8;
constexpr int kDsParts = 8;

template <int D>
__global__ void __launch_bounds__(256) gla_gdn_tail_reduce_kernel(float* partial,
                                                                  const float* mpartial,
                                                                  uint8_t* mtail, WorkPlan wp) {
  static_assert(D == 128 && D / 8 == 2 * kGramParts, "two K chunks of 128 rows per block");
  constexpr int PF = IncCfg<D>::kPartialFloats;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t t = blockIdx.x;
  const int64_t u = static_cast<int64_t>(wp.full_units()) + t;
  int32_t c0, c1;
  wp.slot_range(u, c0, c1);
  if (blockIdx.y < kGramParts) {
    const int i = threadIdx.x & 127;                        // row of M_f
    const int ch = 2 * blockIdx.y + (threadIdx.x >> 7);     // elements 8 ch .. 8 ch + 7
    float x[8];
    const float* src = mpartial + (u + c0) * static_cast<int64_t>(D) * D + ch * 8 * D + i;
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = src[e * D];
    for (int cc = c0 + 1; cc <= c1; ++cc) {
      src += static_cast<int64_t>(D) * D;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] += src[e * D];
    }
    uint4 hi, lo;
    split_bf16x8(x, hi, lo);
    uint8_t* img = mtail + t * (2 * GramImage<D>::kBytes);
    const int off = GramImage<D>::offset(i, ch);
    *reinterpret_cast<uint4*>(img + off) = hi;
    *reinterpret_cast<uint4*>(img + GramImage<D>::kBytes + off) = lo;
  } else if (c1 > c0) {
    float4* dst = reinterpret_cast<float4*>(partial + (u + c0) * PF);
    for (int x = (blockIdx.y - kGramParts) * blockDim.x + threadIdx.x; x < PF / 4;
         x += kDsParts * blockDim.x) {
      float4 acc = dst[x];
      for (int cc = c0 + 1; cc <= c1; ++cc) {
        const float4 v = reinterpret_cast<const float4*>(partial + (u + cc) * PF)[x];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      dst[x] = acc;
    }
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Tensor-core delta scan (d = 128).  Same recurrence as gla_gdn_scan_kernel;
// the per-frame product M_f S_{f-1}[:, J] of a block's column group J runs on
// tcgen05 with a bf16 hi/lo split of both factors, Mh Sh + Mh Sl + Ml Sh in
// fp32 (the dropped Ml Sl term is ~2^-16 relative): one product of Mh with
// [Sh | Sl] (N = 48 + the group's padded width) into TMEM columns
// [0, 48 + N) and Ml Sh accumulated onto columns [0, N), 16 MMAs per frame;
// the consumers add columns j and 48 + j:
//   A = M_f hi / lo   [M = 128 rows i, K = 128]  K-major, no swizzle: the
//                     GramImage pair that the increment kernel (whole units)
//                     or the tail reduction wrote, bulk-copied as it is
//   B = S_{f-1} hi / lo [N = group columns padded to 16, K = 128 rows k]
//                     MN-major, 32-byte swizzle atoms of 16 columns
// A producer warp streams each frame's A images and the group's dS_f rows
// into a two-stage ring; one thread issues the MMAs once the frame's stage has
// landed and the consumers have written B.  Thread i of the four consumer
// warps owns row i of the group's state (TMEM lane i): it reads back row i of
// the product, updates its fp32 state row, writes the next frame's B operand
// (the only step between two products) and then, while the next product
// runs, the bf16 image of S_f^T that the output kernel reads.
template <int D>
struct GdnTcCfg {
  static_assert(D == 128, "tensor-core delta scan is built for d = 128");
  static constexpr int kMaxCols = 48;              // three blocks cover d + 1 columns
  static constexpr int kConsumers = 128;
  static constexpr int kThreads = kConsumers + 64; // + producer warp + MMA warp
  static constexpr int kAImgBytes = GramImage<D>::kBytes;  // one bf16 image (hi or lo)
  static constexpr int kDsBytes = kMaxCols * D * 4;        // the group's dS_f rows, fp32
  static constexpr int kHdrOff = 2 * kAImgBytes + kDsBytes;
  static constexpr int kStageBytes = kHdrOff + 1024;       // + header; stages 1024-aligned
  static constexpr int kStages = 2;                // frame f+1 streams in during frame f
  static constexpr int kBAtomBytes = D * 32;       // 16 columns x 128 rows
  static constexpr int kBImgBytes = (kMaxCols / 16) * kBAtomBytes;
  static constexpr int kTmemCols = 128;            // [Mh Sh + Ml Sh | Mh Sl], 48 + 48 columns
  static constexpr int kBarCount = 2 * kStages + 3;
  static constexpr int kSmemBytes =
      1024 + kStages * kStageBytes + 2 * kBImgBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
};

template <int D>
__global__ void __launch_bounds__(192, 1) gla_gdn_scan_tc_kernel(const GdnScanParams p) {
  using G = Geo<D>;
  using C = GdnTcCfg<D>;
  constexpr int PF = IncCfg<D>::kPartialFloats;
  constexpr unsigned kCode = 64u;
  constexpr int S = C::kStages;
  constexpr int MC = C::kMaxCols;
  constexpr int CPA = G::kAtomElems / 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  // stage s: [A hi | A lo | dS rows | header]
  auto stage = [&](int s) { return smem + s * C::kStageBytes; };
  auto dsst = [&](int s) { return reinterpret_cast<const float*>(stage(s) + 2 * C::kAImgBytes); };
  auto hdr = [&](int s) { return reinterpret_cast<GdnStageHeader*>(stage(s) + C::kHdrOff); };
  const uint32_t b_hi = sbase + S * C::kStageBytes;
  const uint32_t b_lo = b_hi + C::kBImgBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + 2 * C::kBImgBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto mfull = [&](int s) { return bar0 + 8u * s; };        // frame's stage landed (producer)
  auto mempty = [&](int s) { return bar0 + 8u * (S + s); }; // stage used up (4 consumer warps)
  const uint32_t bready = bar0 + 8u * (2 * S);      // B operand of a frame written (4 warps)
  const uint32_t accfull = bar0 + 8u * (2 * S + 1); // product in TMEM (MMA commit)
  const uint32_t done_bar = bar0 + 8u * (2 * S + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.groups;
  const int grp = blockIdx.x % p.groups;
  const int j0 = grp * p.cols;
  const int ncols = (D + 1 - j0 < p.cols) ? D + 1 - j0 : p.cols;
  const int np = (ncols + 15) & ~15;  // MMA N
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t u0 = static_cast<int64_t>(b) * p.F * p.H + h;
  const int64_t srow = static_cast<int64_t>(bh) * D * (D + 1);
  const bool stream = p.tpu > 0 && p.F > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(mfull(s), 1);
      mbar_init(mempty(s), 4);
    }
    mbar_init(bready, 4);
    mbar_init(accfull, 1);
    mbar_init(done_bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  {
    // zero the B operands (columns past the group's stay zero)
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int o = threadIdx.x * 16; o < 2 * C::kBImgBytes; o += C::kThreads * 16)
      st_shared_v4(b_hi + o, z);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    // The whole warp loads the gate and write-strength logits of 32 frames at
    // a time (one lane per frame); lane 0 streams the stages.
    asm volatile("griddepcontrol.wait;" ::: "memory");  // Gram images and dS partials
    if (stream) {
      const uint32_t ds_bytes = static_cast<uint32_t>(ncols) * D * 4;
      float gl = 0.f, bl = 0.f;
      int f = 0;
      for (; f < p.F; ++f) {
        if ((f & 31) == 0) {
          const int ff = f + lane;
          gl = ff < p.F ? __ldg(p.gate + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
          bl = ff < p.F ? __ldg(p.beta + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
        }
        const float g = __shfl_sync(0xffffffffu, gl, f & 31);
        const float bb = __shfl_sync(0xffffffffu, bl, f & 31);
        int ok = 1;
        if (lane == 0) {
          const int s = f % S;
          ok = mbar_wait(mempty(s), static_cast<uint32_t>(((f / S) & 1) ^ 1), abort, kCode) ? 1 : 0;
          if (ok) {
            const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
            int32_t c0, c1;
            p.wp.slot_range(u, c0, c1);
            GdnStageHeader* hd = hdr(s);
            hd->c0 = c0;
            hd->c1 = c1;
            hd->a = 1.0f / (1.0f + expf(-g));
            hd->beta = 1.0f / (1.0f + expf(-bb));
            const int32_t uf = p.wp.full_units();
            const void* aimg =
                u < uf ? static_cast<const void*>(p.mpartial + u * static_cast<int64_t>(D) * D)
                       : static_cast<const void*>(p.mtail + (u - uf) * (2 * C::kAImgBytes));
            mbar_arrive_expect_tx(mfull(s), 2 * C::kAImgBytes + ds_bytes);
            bulk_load(smem_u32(stage(s)), aimg, 2 * C::kAImgBytes, mfull(s));
            bulk_load(smem_u32(stage(s)) + 2 * C::kAImgBytes,
                      p.partial + (u + c0) * PF + static_cast<int64_t>(j0) * D, ds_bytes,
                      mfull(s));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (lane == 0)
        for (int k = (f > S ? f - S : 0); k < f; ++k)
          mbar_wait_drain(mfull(k % S), static_cast<uint32_t>((k / S) & 1));
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && stream) {
      // [Sh | Sl] is one MN-major operand: Sl's atoms follow Sh's 48 columns
      static_assert(C::kBImgBytes == (MC / 16) * C::kBAtomBytes, "B hi / lo adjacent");
      const uint32_t idesc_w = idesc_bf16_f32(128, MC + np, false, true);
      const uint32_t idesc = idesc_bf16_f32(128, np, false, true);
      int f = 0;
      for (; f < p.F; ++f) {
        const int s = f % S;
        if (!mbar_wait(mfull(s), static_cast<uint32_t>((f / S) & 1), abort, kCode)) break;
        if (!mbar_wait(bready, static_cast<uint32_t>(f & 1), abort, kCode)) break;
        tc_fence_after();
        const uint32_t a_hi = smem_u32(stage(s));
        const uint32_t a_lo = a_hi + C::kAImgBytes;
        // Mh [Sh | Sl], then Ml Sh onto the first columns, K = 128 (8 steps of 16)
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const uint32_t abase = pass == 1 ? a_lo : a_hi;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            using GI = GramImage<D>;
            const uint64_t ad = smem_desc(abase + kk * 2 * GI::kChunkStride, GI::kChunkStride,
                                          GI::kGroupStride, kLayoutNone);
            const uint64_t bd = smem_desc(b_hi + kk * 512, C::kBAtomBytes, 256, kLayoutSW32);
            mma_bf16(tmem, ad, bd, pass == 0 ? idesc_w : idesc, (pass > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(accfull);
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else if (warp < 4) {
    // --------------------------------------------------------------- consumers
    const int i = threadIdx.x;  // state row / TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float sr[MC];  // row i of the group's columns of the state, fp32
    // B operand element (k = i, column jl): atom jl / 16, 32-byte row i,
    // 16-byte chunk (jl % 16) / 8 swizzled with bit 2 of the row
    auto b_off = [&](int jl) {
      return (jl >> 4) * C::kBAtomBytes + i * 32 + ((((jl >> 3) & 1) ^ ((i >> 2) & 1)) << 4);
    };
    auto write_b = [&]() {  // the group's columns of row i, hi and lo, then hand B over
#pragma unroll
      for (int jc = 0; jc < MC; jc += 8) {
        if (jc < np) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = (jc + e < ncols) ? sr[jc + e] : 0.f;
          uint4 hi, lo;
          split_bf16x8(x, hi, lo);
          st_shared_v4(b_hi + b_off(jc), hi);
          st_shared_v4(b_lo + b_off(jc), lo);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bready);
    };
    // S_{-1}: row i of the group's columns
#pragma unroll
    for (int jl = 0; jl < MC; ++jl)
      sr[jl] = (jl < ncols && p.state_in != nullptr)
                   ? p.state_in[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jl]
                   : 0.f;
    if (stream) write_b();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int f = 0; f < p.F; ++f) {
      const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
      float a;
      if (stream) {
        const int s = f % S;
        if (!warp_wait(mfull(s), static_cast<uint32_t>((f / S) & 1), abort, kCode)) break;
        const GdnStageHeader hd = *hdr(s);
        a = hd.a;
        const float beta = hd.beta;
        // this frame's dS rows, read while the product runs
        const float* dss = dsst(s);
        float ds[MC];
#pragma unroll
        for (int jl = 0; jl < MC; ++jl) ds[jl] = jl < ncols ? dss[jl * D + i] : 0.f;
        if (!warp_wait(accfull, static_cast<uint32_t>(f & 1), abort, kCode)) break;
        tc_fence_after();
        {
          // (M S)[i, jl] = (Mh Sh + Ml Sh)[i, jl] + (Mh Sl)[i, jl], columns jl and MC + jl
          uint32_t r0[32], r1[32];
          tmem_ld_32cols(tmem + lane_base, r0);
          tmem_ld_32cols(tmem + lane_base + MC, r1);
          tmem_wait_ld();
#pragma unroll
          for (int jl = 0; jl < 32; ++jl)
            if (jl < ncols) {
              const float ms = __uint_as_float(r0[jl]) + __uint_as_float(r1[jl]);
              sr[jl] = a * fmaf(-beta, ms, sr[jl]) + beta * ds[jl];
            }
        }
        {
          uint32_t r0[16], r1[16];
          tmem_ld_16cols(tmem + lane_base + 32, r0);
          tmem_ld_16cols(tmem + lane_base + MC + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int jl = 32; jl < MC; ++jl)
            if (jl < ncols) {
              const float ms = __uint_as_float(r0[jl - 32]) + __uint_as_float(r1[jl - 32]);
              sr[jl] = a * fmaf(-beta, ms, sr[jl]) + beta * ds[jl];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(mempty(s));  // A consumed (product done), dS read
        if (f + 1 < p.F) write_b();             // next frame's B: the product may start
      } else {
        a = 1.0f / (1.0f + expf(-__ldg(p.gate + u)));  // no tokens: the state only decays
#pragma unroll
        for (int jl = 0; jl < MC; ++jl) sr[jl] *= a;
      }
      // bf16 image of S_f^T: row j = j0 + jl, element i
      if (p.image != nullptr) {
        uint16_t* img = reinterpret_cast<uint16_t*>(p.image + u * G::kImageBytes);
        const int ci = i / 8;
#pragma unroll
        for (int jl = 0; jl < MC; ++jl) {
          if (jl < ncols) {
            const int j = j0 + jl;
            const int64_t off = (ci / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                                G::swz(j, ci % CPA) * 16 + (i % 8) * 2;
            img[off / 2] = static_cast<uint16_t>(pack_bf16x2(sr[jl], 0.f) & 0xFFFFu);
          }
        }
      }
    }
    if (p.state_out != nullptr) {
#pragma unroll
      for (int jl = 0; jl < MC; ++jl)
        if (jl < ncols) p.state_out[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jl] = sr[jl];
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gla
