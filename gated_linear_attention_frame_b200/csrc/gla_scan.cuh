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
//     output kernel bulk-copies into shared memory as its B operand.
// After the last frame it writes state_out in the caller's [d][d+1] layout.
// Each thread keeps the partial loads of its next kAhead frames (up to two
// partials per frame, the common case) in flight in registers, issued before
// the current frame is consumed.  Which increment CTAs hold a unit's partials
// is tabulated once per block and chunk of frames in shared memory.  state_in
// and state_out, stored [d][d+1] by the caller, are moved through a shared-
// memory tile so that global accesses are row-contiguous.
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
  WorkPlan wp;             // increment kernel's tile assignment (valid if tpu > 0)
  int H, F, tpu;
};

template <int D>
struct ScanCfg {
  static constexpr int kOcts = D / 8;                          // 8-float chunks per state row
  static constexpr int kBlock = 256;
  static constexpr int kRows = kBlock / kOcts;                  // state rows per block
  static constexpr int kGroups = (D + 1 + kRows - 1) / kRows;   // blocks per (b, h)
  static constexpr int kChunk = 256;                            // frames tabulated at once
};

__device__ __forceinline__ void add8(float (&acc)[8], const float4& a, const float4& b) {
  acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
  acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
}

// Grid: kGroups blocks of 256 threads per (b, h), flattened; block g owns
// state rows j in [g*kRows, (g+1)*kRows) (row d = normaliser).  Launched as a
// programmatic dependent of the increment kernel: only caller inputs
// (state_in, gate logits) are read before griddepcontrol.wait.
template <int D, int kAhead>
__global__ void __launch_bounds__(256, (kAhead <= 2) ? 3 : 2) gla_scan_kernel(const ScanParams p) {
  using G = Geo<D>;
  using C = ScanCfg<D>;
  constexpr int PF = IncCfg<D>::kPartialFloats;
  __shared__ int2 slot_tab[C::kChunk];  // per frame: slots u + x .. u + y of the unit
  __shared__ __align__(16) float st[C::kRows][D + 1];      // state tile [j - j0][i]

  const int bh = blockIdx.x / C::kGroups;
  const int j0 = (blockIdx.x % C::kGroups) * C::kRows;
  const int r = threadIdx.x / C::kOcts;
  const int c = threadIdx.x % C::kOcts;  // key features 8c .. 8c+7
  const int j = j0 + r;                  // value column (j == D: normaliser)
  const bool active = j <= D;
  const int nrows = (D + 1 - j0 < C::kRows) ? D + 1 - j0 : C::kRows;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t u0 = static_cast<int64_t>(b) * p.F * p.H + h;  // unit of frame 0; frame f: + f*H
  const int64_t srow = static_cast<int64_t>(bh) * D * (D + 1);  // this (b, h)'s state

  // state_in -> registers, through the shared tile (global reads along j)
  float S[8];
  if (p.state_in != nullptr) {
    for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kBlock) {
      const int jj = idx % C::kRows, i = idx / C::kRows;
      if (jj < nrows) st[jj][i] = p.state_in[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj];
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = active ? st[r][c * 8 + e] : 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = 0.f;
  }

  const float* col = p.partial + static_cast<int64_t>(j) * D + c * 8;
  constexpr int CPA = G::kAtomElems / 8;
  const int64_t img_off = (c / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                          G::swz(j, c % CPA) * 16;
  const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
  bool waited = false;

  for (int fc = 0; fc < p.F; fc += C::kChunk) {
    const int nf = (p.F - fc < C::kChunk) ? p.F - fc : C::kChunk;
    __syncthreads();  // the previous chunk's table is no longer read
    if (p.tpu > 0) {
      for (int k = threadIdx.x; k < nf; k += C::kBlock) {
        int32_t c0, c1;
        p.wp.slot_range(u0 + static_cast<int64_t>(fc + k) * p.H, c0, c1);
        slot_tab[k] = make_int2(c0, c1);
      }
    }
    __syncthreads();
    if (!waited) {
      asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the increment kernel
      waited = true;
    }
    if (!active) continue;

    // Loads of frame fc + k: slot c0 and, if the unit was split, c0 + 1.
    auto issue = [&](int k, float4 (&x)[4]) {
      if (p.tpu == 0) {
        x[0] = x[1] = x[2] = x[3] = zero4;
        return;
      }
      const int64_t u = u0 + static_cast<int64_t>(fc + k) * p.H;
      const int2 cr = slot_tab[k];
      const float4* s0 = reinterpret_cast<const float4*>(col + (u + cr.x) * PF);
      x[0] = __ldg(s0);
      x[1] = __ldg(s0 + 1);
      if (cr.y > cr.x) {
        x[2] = __ldg(s0 + PF / 4);
        x[3] = __ldg(s0 + PF / 4 + 1);
      } else {
        x[2] = x[3] = zero4;
      }
    };
    float4 x[kAhead][4];
#pragma unroll
    for (int k = 0; k < kAhead; ++k)
      if (k < nf) issue(k, x[k]);
    for (int k0 = 0; k0 < nf; k0 += kAhead) {
#pragma unroll
      for (int kk = 0; kk < kAhead; ++kk) {
        const int k = k0 + kk;
        if (k < nf) {
          const int64_t u = u0 + static_cast<int64_t>(fc + k) * p.H;
          float dS[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          add8(dS, x[kk][0], x[kk][1]);
          add8(dS, x[kk][2], x[kk][3]);
          if (p.tpu > 0) {
            const int2 cr = slot_tab[k];
            for (int cc = cr.x + 2; cc <= cr.y; ++cc) {
              const float4* sx = reinterpret_cast<const float4*>(col + (u + cc) * PF);
              add8(dS, __ldg(sx), __ldg(sx + 1));
            }
          }
          if (k + kAhead < nf) issue(k + kAhead, x[kk]);
          const float g = __ldg(p.gate + u);
          const float a = 1.0f / (1.0f + expf(-g));
#pragma unroll
          for (int e = 0; e < 8; ++e) S[e] = fmaf(a, S[e], dS[e]);
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
  }
  if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (p.state_out != nullptr) {
    __syncthreads();  // every read of the tile (state_in) is done
    if (active) {
#pragma unroll
      for (int e = 0; e < 8; ++e) st[r][c * 8 + e] = S[e];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kBlock) {
      const int jj = idx % C::kRows, i = idx / C::kRows;
      if (jj < nrows) p.state_out[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj] = st[jj][i];
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace gla
