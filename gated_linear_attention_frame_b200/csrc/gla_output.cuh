// gla_output.cuh -- output contraction on tcgen05 tensor cores with the
// normaliser division and the bf16 store fused into the epilogue.
//
// For every token t of frame f (unit u = (b, f, h)) it computes
//   [num | den] = phi(q_t) [S_f[:, :d] | S_f[:, d]],   out_t = num / (den + eps)
// i.e. the block's queries reading the updated cached state, as in the
// SANA-Video talk's block KV cache description.  Per 128-token tile:
//   A = phi(Q tile)   [M = 128 tokens, K = d features]           K-major, TMA
//   B = S_f^T (bf16)  [N = d + 16 rows: d values, normaliser, 15 zero rows]
// S_f^T comes from the scan kernel already laid out as the swizzled
// K-major shared-memory image; one plain bulk copy per swizzle atom loads it,
// once per unit range (double-buffered across units).  The accumulator
// [128 x (d + 16)] fp32 lives in TMEM (two buffers).  The epilogue multiplies
// by the correctly rounded reciprocal of (den + eps), rounds to bf16 (nearest
// even), stages the rows swizzled in shared memory and writes them with TMA
// tensor stores (one 32-row box per epilogue warp; rows past the frame's end
// are clipped by the tensor bounds).
//
// Warp roles: warps 0-3 epilogue, the next kReluWarps ReLU (4; 8 in the
// rotary variant), then one TMA and one MMA warp.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"  // warp_wait
#include "gla_rope.cuh"
#include "sm100_ptx.cuh"

namespace gla {

template <int D, bool kRope = false>
struct OutCfg {
  using G = Geo<D>;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kSBufBytes = G::kAtoms * G::kNPad * G::kRowBytes;  // padded S image
  static constexpr int kStageOutBytes = G::kAtomTileBytes;               // one staging buffer
  static constexpr int kTmemCols = (2 * G::kNPad <= 128) ? 128 : (2 * G::kNPad <= 256) ? 256 : 512;
  static constexpr int kReluWarps = kRope ? 8 : 4;
  static constexpr int kThreads = (kReluWarps + 6) * 32;
  // per-tile normaliser partial sums [token][16-byte chunk of the row]
  static constexpr int kDenRing = kRope ? 2 : 0;
  static constexpr int kDenBytes = kDenRing * kTileTokens * G::kChunksPerRow * 4;
  static constexpr int kBarCount = 3 * kStages + 9 + 2 * kDenRing;
  static constexpr int kSmemBytes = 1024 + kStages * G::kTileBytes + 2 * kSBufBytes +
                                    2 * kStageOutBytes + kDenBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

struct OutParams {
  const uint8_t* image;  // [units][Geo<D>::kImageBytes] bf16 S_f^T images
  float eps;
  WorkPlan wp;           // tile assignment (gridDim.x == wp.G)
  int H, F, T;
  const float* zvec;     // rotary variant: fp32 S_f[:, d] per unit, [units][d]
  RopeGeo rope;          // rotary variant only
};

// kRope: the rotary variant (gla_rope.cuh).  The ReLU warps rotate phi(Q) in
// shared memory for the contraction (only its d value columns are used) and
// form the un-rotated normaliser phi(q_t) . S_f[:, d] from the scan's fp32
// copy of S_f[:, d]: each thread stores the partial dot product of its 8
// features of a token in a [token][chunk] array of a small ring, and the
// epilogue thread of the token adds that row.
template <int D, bool kRope = false>
__global__ void __launch_bounds__(OutCfg<D, kRope>::kThreads, 1)
    gla_output_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_out, const OutParams p) {
  using G = Geo<D>;
  using C = OutCfg<D, kRope>;
  constexpr int R = C::kDenRing;
  constexpr int RW = C::kReluWarps;
  constexpr int kTmaWarp = 4 + RW, kMmaWarp = 5 + RW;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 2u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_base = sbase;
  const uint32_t s_base = q_base + S * G::kTileBytes;
  const uint32_t o_base = s_base + 2 * C::kSBufBytes;
  float* den_ring = reinterpret_cast<float*>(smem + S * G::kTileBytes + 2 * C::kSBufBytes +
                                             2 * C::kStageOutBytes);  // [R][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * G::kTileBytes + 2 * C::kSBufBytes +
                                               2 * C::kStageOutBytes + C::kDenBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto qfull = [&](int s) { return bar0 + 8u * s; };
  auto qrelu = [&](int s) { return bar0 + 8u * (S + s); };
  auto qempty = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto sfull = [&](int b) { return bar0 + 8u * (3 * S + b); };
  auto sempty = [&](int b) { return bar0 + 8u * (3 * S + 2 + b); };
  auto accf = [&](int a) { return bar0 + 8u * (3 * S + 4 + a); };
  auto acce = [&](int a) { return bar0 + 8u * (3 * S + 6 + a); };
  const uint32_t done_bar = bar0 + 8u * (3 * S + 8);
  auto denfull = [&](int m) { return bar0 + 8u * (3 * S + 9 + m); };
  auto denfree = [&](int m) { return bar0 + 8u * (3 * S + 9 + R + m); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto q_buf = [&](int s) { return q_base + s * G::kTileBytes; };
  auto s_buf = [&](int b) { return s_base + b * C::kSBufBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  TileCursor cur;
  cur.init(p.wp, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(qfull(s), 1);
      mbar_init(qrelu(s), RW);
      mbar_init(qempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sempty(b), 1);
      mbar_init(accf(b), 1);
      mbar_init(acce(b), 4);
    }
    mbar_init(done_bar, 1);
    for (int m = 0; m < R; ++m) {
      mbar_init(denfull(m), RW);
      mbar_init(denfree(m), 4);
    }
    *abort = 0;
    fence_mbar_init();
  }
  {
    // Zero the padding rows d+1 .. d+15 of both S buffers (never copied in).
    constexpr int kPadRows = G::kNPad - G::kStateRows;
    constexpr int kPadChunks = 2 * G::kAtoms * kPadRows * (G::kRowBytes / 16);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = threadIdx.x; idx < kPadChunks; idx += C::kThreads) {
      const int ch = idx % (G::kRowBytes / 16);
      const int r = (idx / (G::kRowBytes / 16)) % kPadRows;
      const int blk = idx / ((G::kRowBytes / 16) * kPadRows);  // buffer * kAtoms + atom
      st_shared_v4(s_base + blk * (G::kNPad * G::kRowBytes) + (G::kStateRows + r) * G::kRowBytes +
                       ch * 16,
                   z);
    }
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      int64_t issued = 0, seg = 0;
      bool waited = false;
      int b = 0, f = 0, h = 0;
      for (; cur.valid(); cur.advance(), ++issued) {
        const int64_t u = cur.u;
        const int t = cur.t;
        const int s = static_cast<int>(issued % S);
        if (!mbar_wait(qempty(s), static_cast<uint32_t>(((issued / S) & 1) ^ 1), abort, kCode))
          break;
        if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
        mbar_arrive_expect_tx(qfull(s), G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(q_buf(s) + a * G::kAtomTileBytes, &tm_q, qfull(s), a * G::kAtomElems, h,
                      t * kTileTokens, f, b);
        if (cur.first) {
          if (!waited) {
            // q is a caller input; the state images come from the scan kernel,
            // which this grid may have started alongside.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
          }
          const int sb = static_cast<int>(seg & 1);
          if (!mbar_wait(sempty(sb), static_cast<uint32_t>(((seg >> 1) & 1) ^ 1), abort, kCode))
            break;
          mbar_arrive_expect_tx(sfull(sb), G::kImageBytes);
          const uint8_t* src = p.image + u * static_cast<int64_t>(G::kImageBytes);
#pragma unroll
          for (int a = 0; a < G::kAtoms; ++a)
            bulk_load(s_buf(sb) + a * G::kNPad * G::kRowBytes, src + a * G::kImageAtomBytes,
                      G::kImageAtomBytes, sfull(sb));
          ++seg;
        }
      }
      for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait_drain(qfull(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
      for (int64_t sg = (seg > 2 ? seg - 2 : 0); sg < seg; ++sg)
        mbar_wait_drain(sfull(static_cast<int>(sg & 1)), static_cast<uint32_t>((sg >> 1) & 1));
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, G::kNPad, false, false);
      constexpr int KPA = G::kAtomElems / 16;  // 16-wide K steps per swizzle row
      int64_t i = 0, seg = 0;
      int sb = 0;
      for (; cur.valid(); cur.advance(), ++i) {
        const bool first = cur.first;
        const bool last = cur.last;
        if (first) {
          sb = static_cast<int>(seg & 1);
          if (!mbar_wait(sfull(sb), static_cast<uint32_t>((seg >> 1) & 1), abort, kCode)) break;
        }
        const int ab = static_cast<int>(i & 1);
        if (!mbar_wait(acce(ab), static_cast<uint32_t>(((i >> 1) & 1) ^ 1), abort, kCode)) break;
        const int s = static_cast<int>(i % S);
        if (!mbar_wait(qrelu(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int a = kk / KPA, w = kk % KPA;
          const uint64_t ad = smem_desc(q_buf(s) + a * G::kAtomTileBytes + w * 32, 16,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd = smem_desc(s_buf(sb) + a * G::kNPad * G::kRowBytes + w * 32, 16,
                                        G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + ab * G::kNPad, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(qempty(s));
        mma_commit(accf(ab));
        if (last) {
          mma_commit(sempty(sb));
          ++seg;
        }
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ ReLU
    constexpr int CPR = G::kChunksPerRow;
    constexpr int RPP = RW * 32 / CPR;  // rows per pass of the ReLU warps
    constexpr int kPasses = kTileTokens / RPP;
    constexpr int CPA = G::kAtomElems / 8;
    const int rt = threadIdx.x - 128;
    const int c = rt % CPR;
    const int r0 = rt / CPR;
    const uint32_t off0 =
        (c / CPA) * G::kAtomTileBytes + r0 * G::kRowBytes + G::swz(r0, c % CPA) * 16;
    RopeChunk rc{};
    RopeStep st{};
    int frame = 0;
    float zc[8];  // rotary: S_f[8c .. 8c+7, d] of the current unit
#pragma unroll
    for (int e = 0; e < 8; ++e) zc[e] = 0.f;
    if constexpr (kRope) {
      rc = rope_chunk(p.rope, c);
      rope_step_init(p.rope, c, D / 2, st);
      asm volatile("griddepcontrol.wait;" ::: "memory");  // zvec comes from the scan kernel
    }
    int64_t i = 0;
    for (; cur.valid(); cur.advance(), ++i) {
      const int s = static_cast<int>(i % S);
      if (!warp_wait(qfull(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
      const uint32_t base = q_buf(s) + off0;
      if constexpr (!kRope) {
#pragma unroll
        for (int m = 0; m < kPasses; ++m) {
          const uint32_t addr = base + m * RPP * G::kRowBytes;
          uint4 w = ld_shared_v4(addr);
          relu8(w);
          st_shared_v4(addr, w);
        }
      } else {
        const int mr = static_cast<int>(i % R);
        if (!warp_wait(denfree(mr), static_cast<uint32_t>(((i / R) & 1) ^ 1), abort, kCode)) break;
        if (cur.first) {
          frame = static_cast<int>((cur.u / p.H) % p.F);
          const float4* zp = reinterpret_cast<const float4*>(p.zvec + cur.u * D + c * 8);
          const float4 z0 = __ldg(zp), z1 = __ldg(zp + 1);
          zc[0] = z0.x; zc[1] = z0.y; zc[2] = z0.z; zc[3] = z0.w;
          zc[4] = z1.x; zc[5] = z1.y; zc[6] = z1.z; zc[7] = z1.w;
        }
        RopeRowPos rp;
        rp.start(cur.t * kTileTokens + r0, p.rope.grid_w);
        rope_coeffs(p.rope, rc, frame, rp, p.T, st.cs01, st.cs23);  // first row of the tile
        float* den = den_ring + mr * kTileTokens * CPR;
#pragma unroll
        for (int m = 0; m < kPasses; ++m) {
          const uint32_t addr = base + m * RPP * G::kRowBytes;
          uint4 w = ld_shared_v4(addr);
          relu8(w);
          // normaliser on the un-rotated features; the CPR lanes of a row
          // hold its CPR chunks
          float part = 0.f;
          part = fmaf(bf16lo_to_f32(w.x), zc[0], part);
          part = fmaf(bf16hi_to_f32(w.x), zc[1], part);
          part = fmaf(bf16lo_to_f32(w.y), zc[2], part);
          part = fmaf(bf16hi_to_f32(w.y), zc[3], part);
          part = fmaf(bf16lo_to_f32(w.z), zc[4], part);
          part = fmaf(bf16hi_to_f32(w.z), zc[5], part);
          part = fmaf(bf16lo_to_f32(w.w), zc[6], part);
          part = fmaf(bf16hi_to_f32(w.w), zc[7], part);
          den[(r0 + m * RPP) * CPR + c] = part;
          rotate8(w, st.cs01, st.cs23);
          st_shared_v4(addr, w);
          rope_step_next(st, rp, p.rope.grid_w);
          rp.next(RPP, p.rope.grid_w);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(denfull(mr));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(qrelu(s));
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // token within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    int64_t i = 0;
    int b = 0, f = 0, h = 0;
    for (; cur.valid(); cur.advance(), ++i) {
      const int ab = static_cast<int>(i & 1);
      if (!warp_wait(accf(ab), static_cast<uint32_t>((i >> 1) & 1), abort, kCode)) break;
      tc_fence_after();
      const uint32_t tb = tmem + lane_base + ab * G::kNPad;
      float den;
      if constexpr (kRope) {
        const int mr = static_cast<int>(i % R);
        if (!warp_wait(denfull(mr), static_cast<uint32_t>((i / R) & 1), abort, kCode)) break;
        {
          constexpr int CPR = G::kChunksPerRow;
          const float4* dp = reinterpret_cast<const float4*>(den_ring + (mr * kTileTokens + row) * CPR);
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int x = 0; x < CPR / 4; ++x) {
            const float4 v = dp[x];
            s4[0] += v.x;
            s4[1] += v.y;
            s4[2] += v.z;
            s4[3] += v.w;
          }
          den = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(denfree(mr));
      } else {
        uint32_t dr;
        tmem_ld_1col(tb + D, dr);
        tmem_wait_ld();
        den = __uint_as_float(dr);
      }
      const float rinv = 1.0f / (den + p.eps);
      if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
      const int tok0 = cur.t * kTileTokens + q4 * 32;  // first token of this warp's rows
#pragma unroll
      for (int a = 0; a < G::kAtoms; ++a) {
        const int buf = static_cast<int>((i * G::kAtoms + a) & 1);
        const uint32_t stg = o_base + buf * C::kStageOutBytes;
        if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read smem
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < G::kAtomElems / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(tb + a * G::kAtomElems + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * ch + 0]) * rinv,
                              __uint_as_float(r[8 * ch + 1]) * rinv);
            w.y = pack_bf16x2(__uint_as_float(r[8 * ch + 2]) * rinv,
                              __uint_as_float(r[8 * ch + 3]) * rinv);
            w.z = pack_bf16x2(__uint_as_float(r[8 * ch + 4]) * rinv,
                              __uint_as_float(r[8 * ch + 5]) * rinv);
            w.w = pack_bf16x2(__uint_as_float(r[8 * ch + 6]) * rinv,
                              __uint_as_float(r[8 * ch + 7]) * rinv);
            st_shared_v4(stg + row * G::kRowBytes + G::swz(row, cc * 4 + ch) * 16, w);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (tok0 < p.T)
            tma_store_5d(&tm_out, stg + q4 * 32 * G::kRowBytes, a * G::kAtomElems, h, tok0, f, b);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce(ab));
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  __syncwarp();  // producer / MMA roles ran on lane 0 only
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace gla
