// gla_scan.cuh -- gated prefix scan of the per-frame state increments.
//
// S_f = a_f * S_{f-1} + dS_f with a_f = 1 / (1 + exp(-g[b, f, h])) and
// S_{-1} = state_in: the cached state of the previous block decayed by the
// frame's gate, plus the block's own contribution (SANA-Video talk, block KV
// cache segment; decay gates from the SANA-WM method components).  The
// recurrence is elementwise in the d x (d+1) state, so the kernel runs one
// thread per (b, h, value row j, chunk of 8 key features) and loops over the
// frames in fp32.  Per frame it
//   * sums the unit's fp32 partial increments written by the increment kernel
//     (one per CTA that owned some of the unit's tiles; rows d..d+3 of a
//     partial are four partial sums of the normaliser column),
//   * updates S in registers,
//   * writes S_f^T rounded to bf16 into the swizzled K-major image that the
//     output kernel bulk-copies into shared memory as its B operand.
// After the last frame it writes state_out in the caller's [d][d+1] layout.
// Loads of the next frames' partials are issued before the current frame's
// update so several frames are in flight per thread.
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
  int H, F, tpu;
  int64_t W;               // increment kernel tiles
  int32_t G;               // increment kernel CTAs
};

// Grid: ceil(NT / 256) blocks of 256 threads per (b, h), flattened.
template <int D>
__global__ void __launch_bounds__(256) gla_scan_kernel(const ScanParams p) {
  using G = Geo<D>;
  constexpr int CPR = D / 8;
  constexpr int NT = (D + 1) * CPR;  // threads per (b, h)
  constexpr int PF = IncCfg<D>::kPartialFloats;
  constexpr int kBlocksPerBH = (NT + 255) / 256;
  const int bh = blockIdx.x / kBlocksPerBH;
  const int tid = (blockIdx.x % kBlocksPerBH) * 256 + threadIdx.x;
  if (tid >= NT) return;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int j = tid / CPR;  // value column (j == D: normaliser)
  const int c = tid % CPR;  // key features 8c .. 8c+7
  const TileSplit split{p.W, p.G};

  float S[8];
  if (p.state_in != nullptr) {
    const float* src = p.state_in + (static_cast<int64_t>(bh) * D + c * 8) * (D + 1) + j;
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = src[e * (D + 1)];
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = 0.f;
  }

  // Sum of the partial increments of unit u for this thread's 8 elements.
  auto load_increment = [&](int64_t u, float (&dS)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) dS[e] = 0.f;
    if (p.tpu == 0) return;
    const int64_t c0 = split.owner(u * p.tpu);
    const int64_t c1 = split.owner(u * p.tpu + p.tpu - 1);
    for (int64_t cta = c0; cta <= c1; ++cta) {
      const float* src = p.partial + (u + cta) * PF + c * 8;
      const int nrows = (j < D) ? 1 : 4;
      for (int rr = 0; rr < nrows; ++rr) {
        const float4* s4 = reinterpret_cast<const float4*>(src + static_cast<int64_t>(j + rr) * D);
        const float4 x0 = __ldg(s4);
        const float4 x1 = __ldg(s4 + 1);
        dS[0] += x0.x;
        dS[1] += x0.y;
        dS[2] += x0.z;
        dS[3] += x0.w;
        dS[4] += x1.x;
        dS[5] += x1.y;
        dS[6] += x1.z;
        dS[7] += x1.w;
      }
    }
  };

  constexpr int CPA = G::kAtomElems / 8;
  const int64_t img_off = (c / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                          G::swz(j, c % CPA) * 16;

  constexpr int kAhead = 4;  // frames of increments in flight per thread
  float pre[kAhead][8];
#pragma unroll
  for (int k = 0; k < kAhead; ++k) {
    if (k < p.F) load_increment((static_cast<int64_t>(b) * p.F + k) * p.H + h, pre[k]);
  }
  for (int f0 = 0; f0 < p.F; f0 += kAhead) {
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      const int f = f0 + k;
      if (f < p.F) {
        const int64_t u = (static_cast<int64_t>(b) * p.F + f) * p.H + h;
        const float g = __ldg(p.gate + u);
        const float a = 1.0f / (1.0f + expf(-g));
#pragma unroll
        for (int e = 0; e < 8; ++e) S[e] = fmaf(a, S[e], pre[k][e]);
        if (f + kAhead < p.F)
          load_increment((static_cast<int64_t>(b) * p.F + f + kAhead) * p.H + h, pre[k]);
        if (p.image != nullptr) {
          uint4 w;
          w.x = pack_bf16x2(S[0], S[1]);
          w.y = pack_bf16x2(S[2], S[3]);
          w.z = pack_bf16x2(S[4], S[5]);
          w.w = pack_bf16x2(S[6], S[7]);
          *reinterpret_cast<uint4*>(p.image + u * G::kImageBytes + img_off) = w;
        }
      }
    }
  }

  if (p.state_out != nullptr) {
    float* dst = p.state_out + (static_cast<int64_t>(bh) * D + c * 8) * (D + 1) + j;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e * (D + 1)] = S[e];
  }
}

}  // namespace gla
