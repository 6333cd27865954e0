// gla_scan_bwd.cuh -- reverse gated scan of the backward pass.
//
// The forward recurrence S_f = a_f S_{f-1} + dS_f (SANA-Video talk, block KV
// cache: each block adds its contribution to the decayed cached state) has
// the adjoint recurrence, frames in descending order,
//   G_f = L_f + a_{f+1} G_{f+1},   G_{F-1} = L_{F-1} + dstate_out,
// where L_f = sum_{t in f} phi(q_t)^T [dnum_t | dden_t] is frame f's local
// state gradient (written by the query-side backward kernel as partials, in
// the same slot layout as the forward increments) and G_f is the total
// gradient reaching S_f.  From it:
//   da_f = <G_f, S_{f-1}>  (S_{-1} = state_in),   dstate_in = a_0 G_0,
// and G_f^T is written for the key/value backward kernel as two bf16 images
// in the swizzled K-major layout of the forward prefix states, G = G_hi +
// G_lo with G_hi = bf16(G) and G_lo = bf16(G - G_hi) (value rows 0..d-1), plus
// the normaliser row G_f[:, d] in fp32: dk = [v | 1] G^T cancels strongly
// when a frame has few tokens (out_t then stays near v_t and dk carries
// dout_t . (v_t - out_t)), so a single bf16 copy of G is not accurate enough.
//
// Same structure as the forward scan: a producer warp bulk-copies each
// frame's partials and S_{f-1} rows (the forward states saved by the
// recompute pass) into a ring of shared-memory stages, eight consumer warps
// update G in fp32.  da_f is reduced per warp and written as 8 partial sums
// per (unit, block); gla_dgate_kernel adds them in a fixed order.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"
#include "gla_scan.cuh"
#include "sm100_ptx.cuh"

namespace gla {

struct ScanBwdParams {
  const float* partial;     // local state gradients L_f (slots as the forward increments)
  const float* gate;        // [B, F, H]
  const float* states;      // forward S_f^T per unit, [units][d+1][d] fp32
  const float* state_in;    // [B, H, d, d+1] or nullptr
  const float* dstate_out;  // [B, H, d, d+1] or nullptr
  float* dstate_in;         // [B, H, d, d+1] or nullptr
  uint8_t* image;           // G_f^T images (hi part) [units][kImageBytes], rows 0..d-1
  uint8_t* image_lo;        // G_f^T images (lo part) [units][kImageBytes], rows 0..d-1
  float* gnorm;             // G_f[:, d] in fp32 [units][d]
  float* da_part;           // [units][kGroups][8] per-warp partial sums of da_f
  WorkPlan wp;
  int H, F, tpu;
};

template <int D>
struct ScanBwdCfg {
  using SC = ScanCfg<D, 3>;
  static constexpr int kStages = 3;
  static constexpr int kRows = SC::kRows;
  static constexpr int kGroups = SC::kGroups;
  static constexpr int kThreads = SC::kThreads;
  static constexpr int kConsumers = SC::kConsumers;
  static constexpr int kSlotBytes = SC::kSlotBytes;
  // two partial slots + the S_{f-1} rows + header
  static constexpr int kStageBytes = 3 * kSlotBytes + 16;
  static constexpr int kTileBytes = kRows * (D + 1) * 4;
  static constexpr int kSmemBytes = 128 + kStages * kStageBytes + 2 * kTileBytes + 2 * kStages * 8 + 16;
  static_assert(2 * kSmemBytes <= 228 * 1024, "two blocks per SM");
};

struct BwdStageHeader {
  int32_t c0, c1;  // slots of the unit's local-gradient partials: u + c0 .. u + c1
  float a_next;    // a_{f+1} (1 for the last frame)
  int32_t has_prev;  // S_{f-1} rows were copied (f > 0)
};

template <int D>
__global__ void __launch_bounds__(288, 2) gla_scan_bwd_kernel(const ScanBwdParams p) {
  using G = Geo<D>;
  using C = ScanBwdCfg<D>;
  constexpr int PF = IncCfg<D>::kPartialFloats;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 8u;
  constexpr int kCW = 8;
  constexpr int kOcts = D / 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  auto stage = [&](int s) { return smem + s * C::kStageBytes; };  // [L0 | L1 | S_prev | hdr]
  float(*st)[D + 1] = reinterpret_cast<float(*)[D + 1]>(smem + S * C::kStageBytes);  // state_in
  float(*gt)[D + 1] =
      reinterpret_cast<float(*)[D + 1]>(smem + S * C::kStageBytes + C::kTileBytes);  // dstate
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + 2 * C::kTileBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  volatile int* abort = reinterpret_cast<volatile int*>(bars + 2 * S);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / C::kGroups;
  const int grp = blockIdx.x % C::kGroups;
  const int j0 = grp * C::kRows;
  const int nrows = (D + 1 - j0 < C::kRows) ? D + 1 - j0 : C::kRows;
  const int r = threadIdx.x / kOcts;
  const int c = threadIdx.x % kOcts;
  const int j = j0 + r;
  const bool consumer = warp < kCW;
  const bool active = consumer && r < nrows;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int64_t u0 = static_cast<int64_t>(b) * p.F * p.H + h;
  const int64_t srow = static_cast<int64_t>(bh) * D * (D + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kCW);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const bool stream = p.tpu > 0 && p.F > 0;
  float G8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float Sin8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (warp == kCW) {
    // ---------------------------------------------------------------- producer
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (stream) {
      const uint32_t bytes = static_cast<uint32_t>(nrows) * D * 4;
      float gl = 0.f;
      int n = 0;  // frames issued, in descending order f = F-1-n
      for (; n < p.F; ++n) {
        const int f = p.F - 1 - n;
        // lane l holds the gate logit of frame (F - 1 - (n & ~31) - l) + 1, i.e.
        // a_{f+1} for this chunk of 32 descending frames
        if ((n & 31) == 0) {
          const int ff = f + 1 - lane;
          gl = (ff >= 1 && ff < p.F) ? __ldg(p.gate + u0 + static_cast<int64_t>(ff) * p.H) : 0.f;
        }
        const float g_next = __shfl_sync(0xffffffffu, gl, n & 31);
        int ok = 1;
        if (lane == 0) {
          const int s = n % S;
          ok = mbar_wait(empty(s), static_cast<uint32_t>(((n / S) & 1) ^ 1), abort, kCode) ? 1 : 0;
          if (ok) {
            const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
            int32_t c0, c1;
            p.wp.slot_range(u, c0, c1);
            BwdStageHeader* hdr =
                reinterpret_cast<BwdStageHeader*>(stage(s) + 3 * C::kSlotBytes);
            hdr->c0 = c0;
            hdr->c1 = c1;
            hdr->a_next = (f == p.F - 1) ? 1.0f : 1.0f / (1.0f + expf(-g_next));
            hdr->has_prev = f > 0 ? 1 : 0;
            const float* src = p.partial + (u + c0) * PF + static_cast<int64_t>(j0) * D;
            uint32_t tx = (c1 > c0 ? 2u : 1u) * bytes + (f > 0 ? bytes : 0u);
            mbar_arrive_expect_tx(full(s), tx);
            bulk_load(smem_u32(stage(s)), src, bytes, full(s));
            if (c1 > c0) bulk_load(smem_u32(stage(s)) + C::kSlotBytes, src + PF, bytes, full(s));
            if (f > 0)
              bulk_load(smem_u32(stage(s)) + 2 * C::kSlotBytes,
                        p.states + (u - p.H) * PF + static_cast<int64_t>(j0) * D, bytes, full(s));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (lane == 0)
        for (int k = (n > S ? n - S : 0); k < n; ++k)
          mbar_wait_drain(full(k % S), static_cast<uint32_t>((k / S) & 1));
    }
  } else {
    // --------------------------------------------------------------- consumers
    // dstate_out and state_in through shared tiles (caller layout [d][d+1]).
    if (p.dstate_out != nullptr || p.state_in != nullptr) {
      for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kConsumers) {
        const int jj = idx % C::kRows, i = idx / C::kRows;
        if (jj < nrows) {
          const int64_t off = srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj;
          gt[jj][i] = p.dstate_out != nullptr ? p.dstate_out[off] : 0.f;
          st[jj][i] = p.state_in != nullptr ? p.state_in[off] : 0.f;
        }
      }
      named_bar_sync(1, C::kConsumers);
      if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          G8[e] = gt[r][c * 8 + e];
          Sin8[e] = st[r][c * 8 + e];
        }
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const float* gcol = p.partial + static_cast<int64_t>(j) * D + c * 8;
    constexpr int CPA = G::kAtomElems / 8;
    const int64_t img_off = (c / CPA) * G::kImageAtomBytes + j * G::kRowBytes +
                            G::swz(j, c % CPA) * 16;
    for (int n = 0; n < p.F; ++n) {
      const int f = p.F - 1 - n;
      const int64_t u = u0 + static_cast<int64_t>(f) * p.H;
      float L[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float Sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float a_next = 1.0f;
      if (stream) {
        const int s = n % S;
        if (!warp_wait(full(s), static_cast<uint32_t>((n / S) & 1), abort, kCode)) break;
        const BwdStageHeader hd =
            *reinterpret_cast<const BwdStageHeader*>(stage(s) + 3 * C::kSlotBytes);
        a_next = hd.a_next;
        if (active) {
          const float4* x = reinterpret_cast<const float4*>(stage(s) + r * D * 4 + c * 32);
          add8(L, x[0], x[1]);
          if (hd.c1 > hd.c0) {
            const float4* y =
                reinterpret_cast<const float4*>(stage(s) + C::kSlotBytes + r * D * 4 + c * 32);
            add8(L, y[0], y[1]);
            for (int cc = hd.c0 + 2; cc <= hd.c1; ++cc) {
              const float4* z = reinterpret_cast<const float4*>(gcol + (u + cc) * PF);
              add8(L, __ldg(z), __ldg(z + 1));
            }
          }
          if (hd.has_prev) {
            const float4* sp =
                reinterpret_cast<const float4*>(stage(s) + 2 * C::kSlotBytes + r * D * 4 + c * 32);
            add8(Sp, sp[0], sp[1]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) Sp[e] = Sin8[e];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));
      } else {
        // frames without tokens: no local gradient; S_{f-1} read directly
        a_next = (f == p.F - 1) ? 1.0f : 1.0f / (1.0f + expf(-__ldg(p.gate + u + p.H)));
        if (active) {
          if (f == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) Sp[e] = Sin8[e];
          } else {
            const float4* sp = reinterpret_cast<const float4*>(
                p.states + (u - p.H) * PF + static_cast<int64_t>(j) * D + c * 8);
            add8(Sp, __ldg(sp), __ldg(sp + 1));
          }
        }
      }
      float da = 0.f;
      if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          G8[e] = fmaf(a_next, G8[e], L[e]);
          da = fmaf(G8[e], Sp[e], da);
        }
        if (p.image != nullptr) {
          if (j < D) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hi[e] = pack_bf16x2(G8[2 * e], G8[2 * e + 1]);
              lo[e] = pack_bf16x2(G8[2 * e] - bf16lo_to_f32(hi[e]),
                                  G8[2 * e + 1] - bf16hi_to_f32(hi[e]));
            }
            *reinterpret_cast<uint4*>(p.image + u * G::kImageBytes + img_off) =
                make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(p.image_lo + u * G::kImageBytes + img_off) =
                make_uint4(lo[0], lo[1], lo[2], lo[3]);
          } else {
            float4* gn = reinterpret_cast<float4*>(p.gnorm + u * D + c * 8);
            gn[0] = make_float4(G8[0], G8[1], G8[2], G8[3]);
            gn[1] = make_float4(G8[4], G8[5], G8[6], G8[7]);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
      if (lane == 0) p.da_part[(u * C::kGroups + grp) * kCW + warp] = da;
    }
  }

  if (consumer && p.dstate_in != nullptr) {
    // dstate_in = a_0 G_0
    const float a0 = p.F > 0 ? 1.0f / (1.0f + expf(-__ldg(p.gate + u0))) : 1.0f;
    named_bar_sync(1, C::kConsumers);
    if (active) {
#pragma unroll
      for (int e = 0; e < 8; ++e) gt[r][c * 8 + e] = a0 * G8[e];
    }
    named_bar_sync(1, C::kConsumers);
    for (int idx = threadIdx.x; idx < D * C::kRows; idx += C::kConsumers) {
      const int jj = idx % C::kRows, i = idx / C::kRows;
      if (jj < nrows) p.dstate_in[srow + static_cast<int64_t>(i) * (D + 1) + j0 + jj] = gt[jj][i];
    }
  }
  __syncwarp();
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// dg[b, f, h] = a (1 - a) * (sum of the da partial sums of unit u), a = sigmoid(g).
template <int D>
__global__ void __launch_bounds__(256) gla_dgate_kernel(const float* da_part, const float* gate,
                                                        float* dgate, int64_t units) {
  using C = ScanBwdCfg<D>;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= units) return;
  float da = 0.f;
  for (int k = 0; k < C::kGroups * 8; ++k) da += da_part[u * C::kGroups * 8 + k];
  const float a = 1.0f / (1.0f + expf(-gate[u]));
  dgate[u] = da * a * (1.0f - a);
}

}  // namespace gla
