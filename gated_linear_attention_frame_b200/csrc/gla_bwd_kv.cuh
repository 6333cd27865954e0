// gla_bwd_kv.cuh -- key/value side of the backward pass on tcgen05.
//
// With G_f the total gradient reaching the state S_f (from the reverse scan)
// and S_f = a_f S_{f-1} + phi(K_f)^T [V_f | 1], for every token t of frame f:
//   dk_t = 1[k_t > 0] * ([v_t | 1] G_f^T)      (d outputs)
//   dv_t = phi(k_t) G_f[:, :d]                 (d outputs)
// The reverse scan hands over G_f as two bf16 images of its value rows, G =
// G_hi + G_lo (the scan's swizzled K-major layout), and its normaliser row
// G_f[:, d] in fp32.  Per 128-token tile, two contractions into TMEM:
//   dk~ : A = v        [M = 128 tokens, K = d]  K-major
//         B = G_hi^T, then G_lo^T, read MN-major [N = d key features]
//         (the sum cancels strongly on frames of few tokens, where a single
//         bf16 copy of G would not hold the tolerance); the epilogue adds the
//         fp32 normaliser row, the "| 1" column of [v | 1]
//   dv  : A = phi(k)   [M = 128 tokens, K = d]  K-major (ReLU in smem)
//         B = G_hi^T read K-major                 [N = d value columns]
// The ReLU warps also keep a per-row byte mask of phi(k) > 0 in a small ring
// for the dk epilogue.
// Warp roles as the forward kernels: 0-3 epilogue, 4-7 ReLU/mask, 8 TMA, 9 MMA.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"  // warp_wait, unit_coords
#include "sm100_ptx.cuh"

namespace gla {

template <int D>
struct BwdKVCfg {
  using G = Geo<D>;
  static_assert(D == 128, "the backward kernels are built for d = 128");
  static constexpr int kStages = 2;
  static constexpr int kStageBytes = 2 * G::kTileBytes;                   // v tile + k tile
  static constexpr int kGAtomBytes = D * G::kRowBytes;                   // value rows of one atom
  static constexpr int kGBufBytes = G::kAtoms * kGAtomBytes;             // one part of G^T
  static constexpr int kMaskRing = 4;
  static constexpr int kMaskBytes = kTileTokens * (D / 8);               // one byte per 8 features
  // dk / dv stores: rounds of 32 tokens x 32 features per warp (64-byte
  // swizzle, 2 KB), two buffers per warp
  static constexpr int kRoundCols = 32;
  static constexpr int kRoundBytes = 32 * kRoundCols * 2;
  static constexpr int kStageOutBytes = 4 * 2 * kRoundBytes;
  static constexpr int kTmemCols = 512;                                  // 2 x (dk~ | dv)
  static constexpr int kThreads = 320;
  static constexpr int kBarCount = 3 * kStages + 2 + 4 + 2 * kMaskRing + 1;
  static constexpr int kGNormBytes = 4 * D * 4;  // a private copy of G_f[:, d] per epilogue warp
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 2 * kGBufBytes +
                                    kStageOutBytes + kMaskRing * kMaskBytes + kGNormBytes +
                                    kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

struct BwdKVParams {
  const uint8_t* gimage;     // [units][kImageBytes] bf16 G_f^T images, hi part (rows 0..d-1)
  const uint8_t* gimage_lo;  // [units][kImageBytes] bf16 G_f^T images, lo part (rows 0..d-1)
  const float* gnorm;        // [units][d] G_f[:, d] in fp32
  WorkPlan wp;
  int H, F, T;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    gla_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_dk,
                      const __grid_constant__ CUtensorMap tm_dv, const BwdKVParams p) {
  using G = Geo<D>;
  using C = BwdKVCfg<D>;
  constexpr int S = C::kStages;
  constexpr int R = C::kMaskRing;
  constexpr unsigned kCode = 16u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto v_buf = [&](int s) { return sbase + s * C::kStageBytes; };
  auto k_buf = [&](int s) { return sbase + s * C::kStageBytes + G::kTileBytes; };
  const uint32_t g_hi = sbase + S * C::kStageBytes;
  const uint32_t g_lo = g_hi + C::kGBufBytes;
  const uint32_t o_base = g_lo + C::kGBufBytes;  // output staging: 2 rounds per epilogue warp
  uint8_t* mask_ring = smem + S * C::kStageBytes + 2 * C::kGBufBytes + C::kStageOutBytes;
  float* gnorm_s = reinterpret_cast<float*>(mask_ring + R * C::kMaskBytes);  // [4][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(mask_ring + R * C::kMaskBytes + C::kGNormBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto relu_done = [&](int s) { return bar0 + 8u * (S + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * S + s); };
  const uint32_t gfull = bar0 + 8u * (3 * S);
  const uint32_t gempty = bar0 + 8u * (3 * S + 1);
  auto accf = [&](int a) { return bar0 + 8u * (3 * S + 2 + a); };
  auto acce = [&](int a) { return bar0 + 8u * (3 * S + 4 + a); };
  auto maskfull = [&](int m) { return bar0 + 8u * (3 * S + 6 + m); };
  auto maskfree = [&](int m) { return bar0 + 8u * (3 * S + 6 + R + m); };
  const uint32_t done_bar = bar0 + 8u * (3 * S + 6 + 2 * R);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  TileCursor cur;
  cur.init(p.wp, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(relu_done(s), 4);
      mbar_init(empty(s), 1);
    }
    mbar_init(gfull, 1);
    mbar_init(gempty, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf(a), 1);
      mbar_init(acce(a), 4);
    }
    for (int m = 0; m < R; ++m) {
      mbar_init(maskfull(m), 4);
      mbar_init(maskfree(m), 4);
    }
    mbar_init(done_bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      asm volatile("griddepcontrol.wait;" ::: "memory");  // G images of the reverse scan
      int64_t issued = 0, seg = 0;
      int b = 0, f = 0, h = 0;
      for (; cur.valid(); cur.advance(), ++issued) {
        if (cur.first) {
          unit_coords(cur.u, p.H, p.F, b, f, h);
          if (!mbar_wait(gempty, static_cast<uint32_t>((seg & 1) ^ 1), abort, kCode)) break;
          mbar_arrive_expect_tx(gfull, 2u * C::kGBufBytes);
          const int64_t off = static_cast<int64_t>(cur.u) * G::kImageBytes;
#pragma unroll
          for (int a = 0; a < G::kAtoms; ++a) {
            bulk_load(g_hi + a * C::kGAtomBytes, p.gimage + off + a * G::kImageAtomBytes,
                      C::kGAtomBytes, gfull);
            bulk_load(g_lo + a * C::kGAtomBytes, p.gimage_lo + off + a * G::kImageAtomBytes,
                      C::kGAtomBytes, gfull);
          }
          ++seg;
        }
        const int s = static_cast<int>(issued % S);
        if (!mbar_wait(empty(s), static_cast<uint32_t>(((issued / S) & 1) ^ 1), abort, kCode))
          break;
        const int t = cur.t;
        mbar_arrive_expect_tx(full(s), 2u * G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a) {
          tma_load_5d(v_buf(s) + a * G::kAtomTileBytes, &tm_v, full(s), a * G::kAtomElems, h,
                      t * kTileTokens, f, b);
          tma_load_5d(k_buf(s) + a * G::kAtomTileBytes, &tm_k, full(s), a * G::kAtomElems, h,
                      t * kTileTokens, f, b);
        }
      }
      for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait_drain(full(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
      if (seg > 0) mbar_wait_drain(gfull, static_cast<uint32_t>((seg - 1) & 1));
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_dk = idesc_bf16_f32(128, D, false, true);   // B MN-major
      constexpr uint32_t idesc_dv = idesc_bf16_f32(128, D, false, false);  // B K-major
      constexpr int KPA = G::kAtomElems / 16;
      constexpr uint32_t kGAtom = C::kGAtomBytes;
      int64_t i = 0, seg = 0;
      for (; cur.valid(); cur.advance(), ++i) {
        if (cur.first) {
          if (!mbar_wait(gfull, static_cast<uint32_t>(seg & 1), abort, kCode)) break;
        }
        const int ab = static_cast<int>(i & 1);
        if (!mbar_wait(acce(ab), static_cast<uint32_t>(((i >> 1) & 1) ^ 1), abort, kCode)) break;
        const int s = static_cast<int>(i % S);
        if (!mbar_wait(relu_done(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
        tc_fence_after();
        const uint32_t acc_dk = tmem + ab * 256;
        const uint32_t acc_dv = acc_dk + 128;
        // dk~ = v . (G_hi + G_lo)^T : K over the value columns j
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t gb = part == 0 ? g_hi : g_lo;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc(
                v_buf(s) + (kk / KPA) * G::kAtomTileBytes + (kk % KPA) * 32, 16, G::kGroupBytes,
                G::kLayout);
            const uint64_t bd =
                smem_desc(gb + kk * 2 * G::kGroupBytes, kGAtom, G::kGroupBytes, G::kLayout);
            mma_bf16(acc_dk, ad, bd, idesc_dk, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        // dv = phi(k) . G_hi[:, :d] : K over the key features i
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int a = kk / KPA, w = kk % KPA;
          const uint64_t ad = smem_desc(k_buf(s) + a * G::kAtomTileBytes + w * 32, 16,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd = smem_desc(g_hi + a * kGAtom + w * 32, 16, G::kGroupBytes, G::kLayout);
          mma_bf16(acc_dv, ad, bd, idesc_dv, kk > 0 ? 1u : 0u);
        }
        mma_commit(empty(s));
        mma_commit(accf(ab));
        if (cur.last) {
          mma_commit(gempty);
          ++seg;
        }
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- ReLU on k + sign mask
    constexpr int CPR = G::kChunksPerRow;
    constexpr int RPP = kTileTokens / CPR;
    constexpr int CPA = G::kAtomElems / 8;
    const int rt = threadIdx.x - 128;
    const int c = rt % CPR;
    const int r0 = rt / CPR;
    const uint32_t off0 =
        (c / CPA) * G::kAtomTileBytes + r0 * G::kRowBytes + G::swz(r0, c % CPA) * 16;
    int64_t i = 0;
    for (; cur.valid(); cur.advance(), ++i) {
      const int s = static_cast<int>(i % S);
      const int m = static_cast<int>(i % R);
      if (!warp_wait(full(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
      if (!warp_wait(maskfree(m), static_cast<uint32_t>(((i / R) & 1) ^ 1), abort, kCode)) break;
      const uint32_t base = k_buf(s) + off0;
      uint8_t* mrow = mask_ring + m * C::kMaskBytes;
#pragma unroll
      for (int mm = 0; mm < CPR; ++mm) {
        const uint32_t addr = base + mm * RPP * G::kRowBytes;
        uint4 w = ld_shared_v4(addr);
        relu8(w);
        st_shared_v4(addr, w);
        // bit e set <=> feature 8c+e of this token is positive
        uint32_t bits = 0;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bits |= ((ws[e] & 0x7FFFu) != 0u ? 1u : 0u) << (2 * e);
          bits |= ((ws[e] & 0x7FFF0000u) != 0u ? 1u : 0u) << (2 * e + 1);
        }
        mrow[(r0 + mm * RPP) * (D / 8) + c] = static_cast<uint8_t>(bits);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(relu_done(s));
        mbar_arrive(maskfull(m));
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // token within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // G_f[:, d] of the reverse scan
    int64_t i = 0;
    int b = 0, f = 0, h = 0;
    for (; cur.valid(); cur.advance(), ++i) {
      const int ab = static_cast<int>(i & 1);
      const int m = static_cast<int>(i % R);
      if (!warp_wait(accf(ab), static_cast<uint32_t>((i >> 1) & 1), abort, kCode)) break;
      if (!warp_wait(maskfull(m), static_cast<uint32_t>((i / R) & 1), abort, kCode)) break;
      tc_fence_after();
      float* gw = gnorm_s + q4 * D;  // this warp's copy of the unit's G_f[:, d]
      if (cur.first) {
        unit_coords(cur.u, p.H, p.F, b, f, h);
        __syncwarp();  // the previous unit's reads of the copy are done
        for (int c = lane; c < D / 4; c += 32)
          reinterpret_cast<float4*>(gw)[c] =
              __ldg(reinterpret_cast<const float4*>(p.gnorm + static_cast<int64_t>(cur.u) * D) + c);
        __syncwarp();
      }
      const int tok0 = cur.t * kTileTokens + q4 * 32;
      const float4* gn = reinterpret_cast<const float4*>(gw);
      // the row's sign mask
      const uint4 mk = *reinterpret_cast<const uint4*>(mask_ring + m * C::kMaskBytes + row * (D / 8));
      __syncwarp();
      if (lane == 0) mbar_arrive(maskfree(m));
      const uint32_t mwords[4] = {mk.x, mk.y, mk.z, mk.w};
#pragma unroll
      for (int out = 0; out < 2; ++out) {  // 0: dk (normaliser row added, masked), 1: dv
        const uint32_t tb = tmem + lane_base + ab * 256 + out * 128;
        const CUtensorMap* tm = out == 0 ? &tm_dk : &tm_dv;
#pragma unroll
        for (int cc = 0; cc < D / C::kRoundCols; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(tb + cc * 32, r);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int col8 = cc * 4 + ch;  // 8-feature chunk index
            const uint32_t mb = (mwords[col8 >> 2] >> (8 * (col8 & 3))) & 0xFFu;
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(r[8 * ch + e]);
            if (out == 0) {
              const float4 g0 = gn[2 * col8], g1 = gn[2 * col8 + 1];
              x[0] += g0.x; x[1] += g0.y; x[2] += g0.z; x[3] += g0.w;
              x[4] += g1.x; x[5] += g1.y; x[6] += g1.z; x[7] += g1.w;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (((mb >> e) & 1u) == 0u) x[e] = 0.f;
            }
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) pk[ch * 4 + e2] = pack_bf16x2(x[2 * e2], x[2 * e2 + 1]);
          }
          const int rnd = out * (D / C::kRoundCols) + cc;
          const uint32_t stg = o_base + q4 * 2 * C::kRoundBytes + (rnd & 1) * C::kRoundBytes;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)  // 64-byte swizzle: chunk ch of row lane
            st_shared_v4(stg + lane * 64 + ((ch ^ ((lane >> 1) & 3)) * 16),
                         make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (tok0 < p.T) tma_store_5d(tm, stg, cc * C::kRoundCols, h, tok0, f, b);
            bulk_commit_group();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce(ab));
    }
    if (lane == 0) bulk_wait_group<0>();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace gla
