// gla_scan.cuh -- gated prefix scan of the per-frame state increments.
//
// S_f = a_f * S_{f-1} + dS_f with a_f = 1 / (1 + exp(-g[b, f, h])) and
// S_{-1} = state_in: the cached state of the previous block decayed by the
// frame's gate, plus the block's own contribution (SANA-Video talk, block KV
// cache segment; decay gates from the SANA-WM method components).  The
// recurrence is elementwise in the d x (d+1) state, so the kernel runs one
// thread per (b, h, value row j, 8 consecutive key features) and loops over
// the frames in fp32.  Per frame it
//   * sums the unit's fp32 partial increments written by the increment kernel
//     (one per CTA that owned some of the unit's tiles),
//   * updates S in registers,
//   * writes S_f^T rounded to bf16 into the swizzled K-major image that the
//     output kernel bulk-copies into shared memory as its B operand (and, for
//     the backward pass, the bf16 rounding of the remainder in a second image).
// After the last frame it writes state_out in the caller's [d][d+1] layout.
// A producer warp streams each frame's partial increments into a ring of
// shared-memory stages with plain bulk copies (one copy per partial: the
// block's rows of it are contiguous), so several frames are in flight without
// holding them in registers; eight consumer warps take one stage per frame.
// Which increment CTAs hold a unit's partials, and the frame's decay, travel
// with the stage.
// state_in and state_out, stored [d][d+1] by the caller, are moved through a
// shared-memory tile so that global accesses run along rows.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"
#include "sm100_ptx.cuh"

namespace gla {

struct ScanParams {
  const float* partial;    // increment partials (see gla_increment.cuh); unused if tpu == 0
  const float* gate;       // [B, F, H]
  const float* state_in;   // [B, H, d, d+1] or nullptr
  float* state_out;        // [B, H, d, d+1] or nullptr
  uint8_t* image;          // [units][kImageBytes] or nullptr (no output kernel)
  float* states;           // [units][d+1][d] fp32 S_f^T per frame, or nullptr (backward only)
  WorkPlan wp;             // increment kernel's tile assignment (valid if tpu > 0)
  int H, F, tpu;
  float* zvec;             // [units][d] fp32 S_f[:, d] per frame, or nullptr (rotary variant)
  uint8_t* image_lo;       // [units][kImageBytes] bf16(S_f - bf16(S_f))^T, value rows 0..d-1,
                           // or nullptr (backward: the query kernel's dq contraction)
  int bh0;                 // first (b, h) of the grid (single-frame calls whose whole
                           // units the increment kernel folds: the split ones only)
};

template <int D, int kStagesT = 3>
struct ScanCfg {
  static constexpr int kOcts = D / 8;                          // 8-float chunks per state row
  static constexpr int kConsumerWarps = 8;
  static constexpr int kConsumers = 32 * kConsumerWarps;
  static constexpr int kThreads = kConsumers + 32;              // + 1 producer warp
  static constexpr int kRows = kConsumers / kOcts;              // state rows per block
  static constexpr int kGroups = (D + 1 + kRows - 1) / kRows;   // blocks per (b, h)
  static constexpr int kStages = kStagesT;
  static constexpr int kSlotBytes = kRows * D * 4;              // one partial's rows: 8 KB
  static constexpr int kStageBytes = 2 * kSlotBytes + 16;       // two partials + StageHeader
  static constexpr int kTileBytes = kRows * (D + 1) * 4;        // state_in / state_out tile
  static constexpr int kSmemBytes = 128 + kStages * kStageBytes + kTileBytes + 2 * kStages * 8 + 16;
};

// Header at the end of each stage, written by the producer with the copies.
struct StageHeader {
  int32_t c0, c1;  // the unit's partials are at slots u + c0 .. u + c1
  float a;         // the frame's decay sigmoid(g)
  int32_t pad;
};

__device__ __forceinline__ void add8(float (&acc)[8], const float4& a, const float4& b) {
  acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
  acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
}

// Grid: kGroups blocks of 288 threads per (b, h), flattened; block g owns
// state rows j in [g*kRows, (g+1)*kRows) (row d = normaliser).  Launched as a
// programmatic dependent of the increment kernel: only caller inputs
// (state_in) are read before griddepcontrol.wait.  kStagesT = 1 serves
// single-frame calls (fewer registers and less shared memory: more blocks
// per SM), 3 serves sequences of frames.
template <int D, int kStagesT>
__global__ void __launch_bounds__(288, (kStagesT == 1) ? 4 : 3)
    gla_scan_kernel(const ScanParams p) {
  using G = Geo<D>;
  using C = ScanCfg<D, kStagesT>;
  constexpr int PF = IncCfg<D>::kPartialFloats;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 4u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  auto stage = [&](int s) { return smem + s * C::kStageBytes; };  // [slot0 | slot1 | header]
  float(*st)[D + 1] = reinterpret_cast<float(*)[D + 1]>(smem + S * C::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kTileBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 2 * S);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = p.bh0 + static_cast<int>(blockIdx.x / C::kGroups);
  const int j0 = (blockIdx.x % C::kGroups) * C::kRows;
  const int nrows = (D + 1 - j0 < C::kRows) ? D + 1 - j0 : C::kRows;
  const int r = threadIdx.x / C::kOcts;  // consumer: row within the block
  const int c = threadIdx.x % C::kOcts;  // consumer: key features 8c .. 8c+7
  const int j = j0 + r;                  // value column (j == D: normaliser)
  constexpr int kCW = C::kConsumerWarps;
  const bool consumer = warp < kCW;
  const bool active = consumer && r < nrows;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t u0 = static_cast<int64_t>(b) * p.F * p.H + h;  // unit of frame 0; frame f: + f*H
  const int64_t srow = static_cast<int64_t>(bh) * D * (D + 1);  // this (b, h)'s state

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kCW);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();  // barriers initialised

  const bool stream_partials = p.tpu > 0 && p.F > 0;
  float S8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (warp == kCW) {
    // ---------------------------------------------------------------- producer
    // Starts streaming partials while the consumers load state_in.
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the increment kernel
    if (stream_partials) {
      // The whole warp loads the gate logits of 32 frames at a time (one lane
      // per frame); lane 0 turns each into a = sigmoid(g) and hands it to the
      // consumers in the stage header, so no consumer waits on a gate load.
      const uint32_t bytes = static_cast<uint32_t>(nrows) * D * 4;
      float gl = 0.f;
      int f = 0;
      for (; f < p.F; ++f) {
        if ((f & 31) == 0) {
          const int ff = f + lane;
          gl = ff < p.F ? __ldg(p.gate + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
        }
        const float g = __shfl_sync(0xffffffffu, gl, f & 31);
        int ok = 1;
        if (lane == 0) {
          const int s = f % S;
          ok = mbar_wait(empty(s), static_cast<uint32_t>(((f / S) & 1) ^ 1), abort, kCode) ? 1 : 0;
          if (ok) {
            const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
            int32_t c0, c1;
            p.wp.slot_range(u, c0, c1);
            StageHeader* hdr = reinterpret_cast<StageHeader*>(stage(s) + 2 * C::kSlotBytes);
            hdr->c0 = c0;
            hdr->c1 = c1;
            hdr->a = 1.0f / (1.0f + expf(-g));
            const float* src = p.partial + (u + c0) * PF + static_cast<int64_t>(j0) * D;
            mbar_arrive_expect_tx(full(s), (c1 > c0 ? 2u : 1u) * bytes);
            bulk_load(smem_u32(stage(s)), src, bytes, full(s));
            if (c1 > c0) bulk_load(smem_u32(stage(s)) + C::kSlotBytes, src + PF, bytes, full(s));
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
    if (p.state_in != nullptr) {
      for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kConsumers) {
        const int jj = idx % C::kRows, i = idx / C::kRows;
        if (jj < nrows) st[jj][i] = p.state_in[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj];
      }
      named_bar_sync(1, C::kConsumers);
      if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) S8[e] = st[r][c * 8 + e];
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partials read directly (rare)
    const float* gcol = p.partial + static_cast<int64_t>(j) * D + c * 8;
    constexpr int CPA = G::kAtomElems / 8;
    const int64_t img_off = (c / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                            G::swz(j, c % CPA) * 16;
    for (int f = 0; f < p.F; ++f) {
      const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
      float dS[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float a;
      if (stream_partials) {
        const int s = f % S;
        if (!warp_wait(full(s), static_cast<uint32_t>((f / S) & 1), abort, kCode)) break;
        const StageHeader hd = *reinterpret_cast<const StageHeader*>(stage(s) + 2 * C::kSlotBytes);
        a = hd.a;
        if (active) {
          const int2 cr = make_int2(hd.c0, hd.c1);
          const float4* x = reinterpret_cast<const float4*>(stage(s) + r * D * 4 + c * 32);
          add8(dS, x[0], x[1]);
          if (cr.y > cr.x) {
            const float4* y = reinterpret_cast<const float4*>(stage(s) + C::kSlotBytes +
                                                              r * D * 4 + c * 32);
            add8(dS, y[0], y[1]);
            for (int cc = cr.x + 2; cc <= cr.y; ++cc) {  // rare: unit split over > 2 CTAs
              const float4* z = reinterpret_cast<const float4*>(gcol + (u + cc) * PF);
              add8(dS, __ldg(z), __ldg(z + 1));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));
      } else {
        a = 1.0f / (1.0f + expf(-__ldg(p.gate + u)));  // frames without tokens
      }
      if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) S8[e] = fmaf(a, S8[e], dS[e]);
        if (p.image != nullptr) {
          uint4 w;
          w.x = pack_bf16x2(S8[0], S8[1]);
          w.y = pack_bf16x2(S8[2], S8[3]);
          w.z = pack_bf16x2(S8[4], S8[5]);
          w.w = pack_bf16x2(S8[6], S8[7]);
          *reinterpret_cast<uint4*>(p.image + u * G::kImageBytes + img_off) = w;
          if (p.image_lo != nullptr && j < D) {
            uint4 l;
            l.x = pack_bf16x2(S8[0] - bf16lo_to_f32(w.x), S8[1] - bf16hi_to_f32(w.x));
            l.y = pack_bf16x2(S8[2] - bf16lo_to_f32(w.y), S8[3] - bf16hi_to_f32(w.y));
            l.z = pack_bf16x2(S8[4] - bf16lo_to_f32(w.z), S8[5] - bf16hi_to_f32(w.z));
            l.w = pack_bf16x2(S8[6] - bf16lo_to_f32(w.w), S8[7] - bf16hi_to_f32(w.w));
            *reinterpret_cast<uint4*>(p.image_lo + u * G::kImageBytes + img_off) = l;
          }
        }
        if (p.zvec != nullptr && j == D) {
          float4* dst = reinterpret_cast<float4*>(p.zvec + u * D + c * 8);
          dst[0] = make_float4(S8[0], S8[1], S8[2], S8[3]);
          dst[1] = make_float4(S8[4], S8[5], S8[6], S8[7]);
        }
        if (p.states != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.states + u * PF + static_cast<int64_t>(j) * D +
                                                  c * 8);
          dst[0] = make_float4(S8[0], S8[1], S8[2], S8[3]);
          dst[1] = make_float4(S8[4], S8[5], S8[6], S8[7]);
        }
      }
    }
  }

  if (consumer && p.state_out != nullptr) {
    named_bar_sync(1, C::kConsumers);  // every consumer is done reading the tile
    if (active) {
#pragma unroll
      for (int e = 0; e < 8; ++e) st[r][c * 8 + e] = S8[e];
    }
    named_bar_sync(1, C::kConsumers);
    for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kConsumers) {
      const int jj = idx % C::kRows, i = idx / C::kRows;
      if (jj < nrows) p.state_out[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj] = st[jj][i];
    }
  }
  __syncwarp();
  __syncthreads();  // the producer's copies have landed before the block exits
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gla
