// gla_bwd_q.cuh -- query side of the backward pass on tcgen05.
//
// For the queries of frame f, with S_f the forward prefix state:
//   num_t = phi(q_t) S_f[:, :d],  den_t = phi(q_t) S_f[:, d] + eps,  rden_t = 1 / den_t
//   dnum_t = dout_t rden_t,       dden_t = -(dout_t . num_t) rden_t^2
//   dq_t  = 1[q_t > 0] * (rden_t (dout_t S_f[:, :d]^T) + dden_t S_f[:, d])
//   L_f   = sum_{t in f} phi(q_t)^T [dnum_t | dden_t]     (frame f's state gradient)
// Per 128-token tile, three contractions into TMEM:
//   MMA1  [num | den] = phi(Q) S_f        A = phi(Q) K-major, B = S_f^T image K-major (N = d+16)
//   MMA2  dout S_f[:, :d]^T               A = dout K-major, B = S_hi^T then S_lo^T images MN-major
//   MMA3  L_f += phi(Q)^T D               A = phi(Q) MN-major, B = D MN-major
// dq is formed from dout itself (exact in bf16) against a hi/lo pair of bf16
// copies of S_f (S = S_hi + S_lo, both images written by the recompute
// scan), with the 1/den scale and the normaliser column's term added in fp32
// in the epilogue: in a frame of few tokens the two terms of dq cancel
// almost exactly (out_t stays near v_t), and bf16 copies of D or of S_f in
// this contraction would leave residue above the tolerance.  MMA2 needs only
// dout, so it runs beside MMA1 and the epilogue's D build.
// D = [dnum | dden | 0 ...] is built in shared memory by the epilogue from
// MMA1's result and dout, as a hi/lo pair of bf16 copies (D = D_hi + D_lo):
// the gate gradient <G_f, S_{f-1}> and dk sum thousands of products of L_f
// with random signs, and one bf16 rounding of D would put their error near
// the tolerance.  The producer loads the dout tile by TMA into the D_hi
// buffer itself (same swizzled 128 x d layout); each epilogue thread writes
// its row of D_lo, keeps its row of D_hi in registers until MMA2 has read
// dout, then overwrites its row of dout with it.  D's first d columns sit in
// two 128-byte-swizzled atoms; the dden column and 15 zero columns in a
// 32-byte-swizzled region of 32-byte rows, so that MMA3's N = 16 part is a
// whole swizzle atom; that region holds dden's hi part in its column 0 and
// its lo part in column 1, so one N = 16 MMA per K step gives both
// (L_f[:, d] = their sum).  L_f is accumulated over a unit's tiles and
// written as an fp32 partial in the forward increment's slot layout (row d =
// sum_t phi(q_t) dden_t) for the reverse scan.
// The ReLU warps keep a byte mask of q > 0 for the dq epilogue, so a q stage
// is released as soon as MMA3 has read it.
// Warp roles: 0-3 epilogue, 4-7 ReLU, 8 TMA, 9 MMA.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"  // warp_wait, unit_coords, IncCfg
#include "sm100_ptx.cuh"

namespace gla {

template <int D>
struct BwdQCfg {
  using G = Geo<D>;
  static_assert(D == 128, "the backward kernels are built for d = 128");
  static constexpr int kStages = 2;
  static constexpr int kSBufBytes = G::kAtoms * G::kNPad * G::kRowBytes;  // S_f^T image (hi)
  static constexpr int kSLoAtomBytes = D * G::kRowBytes;                 // value rows of one atom
  static constexpr int kSLoBytes = G::kAtoms * kSLoAtomBytes;            // S_f^T image (lo)
  static constexpr int kDMainBytes = G::kAtoms * G::kAtomTileBytes;       // dnum, 128-byte swizzle
  static constexpr int kDPadBytes = kTileTokens * 32;                     // [dden | 0 x 15], 32-byte swizzle
  // dq stores: rounds of 32 tokens x 32 features per warp (64-byte swizzle,
  // 2 KB), one buffer for each of the eight warps
  static constexpr int kRoundCols = 32;
  static constexpr int kRoundBytes = 32 * kRoundCols * 2;
  static constexpr int kStageOutBytes = 8 * kRoundBytes;
  static constexpr int kMaskRing = 3;
  static constexpr int kMaskBytes = kTileTokens * (D / 8);                // one bit per feature
  static constexpr int kAcc1 = 0;    // [num | den]  : N = d + 16 columns
  static constexpr int kAcc2 = 160;  // dout S^T     : N = d
  static constexpr int kAcc3 = 288;  // L_f          : N = d + 16
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 320;
  static constexpr int kBarCount = 3 * kStages + 12 + 2 * kMaskRing + 1 + 4;
  // half-row dot products [tile parity][column half][token]
  static constexpr int kDotBytes = 2 * 2 * kTileTokens * 4;
  static constexpr int kSmemBytes = 1024 + kStages * G::kTileBytes + kSBufBytes + kSLoBytes +
                                    kDMainBytes + kDPadBytes + kDMainBytes + kStageOutBytes +
                                    kMaskRing * kMaskBytes + kDotBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

struct BwdQParams {
  const uint8_t* image;     // [units][kImageBytes] bf16 S_f^T images (forward recompute)
  const uint8_t* image_lo;  // [units][kImageBytes] their bf16 remainders, value rows 0..d-1
  const float* states;      // [units][d+1][d] fp32 S_f^T (row d: S_f[:, d])
  float* partial;           // L_f partials [(units + G) slots][d + 1][d]
  float eps;
  WorkPlan wp;
  int H, F, T;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    gla_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_dout,
                     const __grid_constant__ CUtensorMap tm_dq, const BwdQParams p) {
  using G = Geo<D>;
  using C = BwdQCfg<D>;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 32u;
  constexpr int PF = IncCfg<D>::kPartialFloats;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto q_buf = [&](int s) { return sbase + s * G::kTileBytes; };
  const uint32_t s_buf = sbase + S * G::kTileBytes;       // S_hi (d + 16 rows per atom)
  const uint32_t s_lo = s_buf + C::kSBufBytes;            // S_lo (d rows per atom)
  const uint32_t d_buf = s_lo + C::kSLoBytes;             // dout, then D_hi
  const uint32_t d_pad = d_buf + C::kDMainBytes;
  const uint32_t l_buf = d_pad + C::kDPadBytes;           // D_lo
  const uint32_t o_base = l_buf + C::kDMainBytes;         // dq staging: 2 rounds per epilogue warp
  uint8_t* mask_ring = smem + (o_base + C::kStageOutBytes - sbase);
  float* dot_x = reinterpret_cast<float*>(mask_ring + C::kMaskRing * C::kMaskBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(mask_ring + C::kMaskRing * C::kMaskBytes +
                                               C::kDotBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto qfull = [&](int s) { return bar0 + 8u * s; };
  auto qrelu = [&](int s) { return bar0 + 8u * (S + s); };
  auto qempty = [&](int s) { return bar0 + 8u * (2 * S + s); };
  const uint32_t sfull = bar0 + 8u * (3 * S + 0);
  const uint32_t sempty = bar0 + 8u * (3 * S + 1);
  const uint32_t acc1_full = bar0 + 8u * (3 * S + 2);
  const uint32_t acc1_free = bar0 + 8u * (3 * S + 3);
  const uint32_t dfull = bar0 + 8u * (3 * S + 4);
  const uint32_t dfree = bar0 + 8u * (3 * S + 5);
  const uint32_t acc2_full = bar0 + 8u * (3 * S + 6);  // MMA2 done: dout read, dout S^T ready
  const uint32_t acc2_free = bar0 + 8u * (3 * S + 7);
  const uint32_t acc3_full = bar0 + 8u * (3 * S + 8);
  const uint32_t acc3_free = bar0 + 8u * (3 * S + 9);
  const uint32_t done_bar = bar0 + 8u * (3 * S + 10);
  constexpr int R = C::kMaskRing;
  auto maskfull = [&](int m) { return bar0 + 8u * (3 * S + 11 + m); };
  auto maskfree = [&](int m) { return bar0 + 8u * (3 * S + 11 + R + m); };
  const uint32_t doutfull = bar0 + 8u * (3 * S + 11 + 2 * R);  // dout tile landed in D_hi
  const uint32_t lfree = bar0 + 8u * (3 * S + 12 + 2 * R);     // MMA3 read D_lo
  // both column halves of lane quarter q wrote their dot products
  auto xbar = [&](int q) { return bar0 + 8u * (3 * S + 13 + 2 * R + q); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  TileCursor cur;
  cur.init(p.wp, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(qfull(s), 1);
      mbar_init(qrelu(s), 4);
      mbar_init(qempty(s), 1);
    }
    for (int m = 0; m < R; ++m) {
      mbar_init(maskfull(m), 4);
      mbar_init(maskfree(m), 8);
    }
    mbar_init(sfull, 1);
    mbar_init(sempty, 1);
    mbar_init(acc1_full, 1);
    mbar_init(acc1_free, 8);
    mbar_init(dfull, 8);
    mbar_init(lfree, 1);
    for (int q = 0; q < 4; ++q) mbar_init(xbar(q), 2);
    mbar_init(dfree, 1);
    mbar_init(doutfull, 1);
    mbar_init(acc2_full, 1);
    mbar_init(acc2_free, 8);
    mbar_init(acc3_full, 1);
    mbar_init(acc3_free, 4);
    mbar_init(done_bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  {
    // zero: the S image's padding rows, and D's pad region (only the chunk
    // holding column 0, dden, is rewritten per tile)
    constexpr int kPadRows = G::kNPad - G::kStateRows;
    constexpr int kPadChunks = G::kAtoms * kPadRows * (G::kRowBytes / 16);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = threadIdx.x; idx < kPadChunks; idx += C::kThreads) {
      const int ch = idx % (G::kRowBytes / 16);
      const int rr = (idx / (G::kRowBytes / 16)) % kPadRows;
      const int at = idx / ((G::kRowBytes / 16) * kPadRows);
      st_shared_v4(s_buf + at * (G::kNPad * G::kRowBytes) + (G::kStateRows + rr) * G::kRowBytes +
                       ch * 16,
                   z);
    }
    for (int o = threadIdx.x * 16; o < C::kDPadBytes; o += C::kThreads * 16)
      st_shared_v4(d_pad + o, z);
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

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_dout);
      asm volatile("griddepcontrol.wait;" ::: "memory");  // S images of the forward recompute
      int64_t issued = 0, seg = 0;
      int b = 0, f = 0, h = 0;
      for (; cur.valid(); cur.advance(), ++issued) {
        if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
        // Order: q, dout, then (at a unit's start) the state images.  The
        // images wait for the previous unit's last MMA3, which waits for D of
        // the previous tile, which the ReLU warps build only after they have
        // ReLU'd this tile's q: q must not queue behind the images.
        const int s = static_cast<int>(issued % S);
        if (!mbar_wait(qempty(s), static_cast<uint32_t>(((issued / S) & 1) ^ 1), abort, kCode))
          break;
        mbar_arrive_expect_tx(qfull(s), G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(q_buf(s) + a * G::kAtomTileBytes, &tm_q, qfull(s), a * G::kAtomElems, h,
                      cur.t * kTileTokens, f, b);
        // dout of this tile into D_hi once the previous tile's MMA3 read D
        if (!mbar_wait(dfree, static_cast<uint32_t>((issued & 1) ^ 1), abort, kCode)) break;
        mbar_arrive_expect_tx(doutfull, G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(d_buf + a * G::kAtomTileBytes, &tm_dout, doutfull, a * G::kAtomElems, h,
                      cur.t * kTileTokens, f, b);
        // the next tile's dout into L2: its load waits for this tile's MMA3,
        // so it is on the tile chain and should not go to HBM
        {
          TileCursor nx = cur;
          nx.advance();
          if (nx.valid()) {
            int nb, nf, nh;
            unit_coords(nx.u, p.H, p.F, nb, nf, nh);
#pragma unroll
            for (int a = 0; a < G::kAtoms; ++a)
              tma_prefetch_5d(&tm_dout, a * G::kAtomElems, nh, nx.t * kTileTokens, nf, nb);
          }
        }
        if (cur.first) {
          if (!mbar_wait(sempty, static_cast<uint32_t>((seg & 1) ^ 1), abort, kCode)) break;
          mbar_arrive_expect_tx(sfull, G::kImageBytes + C::kSLoBytes);
          const int64_t off = static_cast<int64_t>(cur.u) * G::kImageBytes;
#pragma unroll
          for (int a = 0; a < G::kAtoms; ++a) {
            bulk_load(s_buf + a * G::kNPad * G::kRowBytes, p.image + off + a * G::kImageAtomBytes,
                      G::kImageAtomBytes, sfull);
            bulk_load(s_lo + a * C::kSLoAtomBytes, p.image_lo + off + a * G::kImageAtomBytes,
                      C::kSLoAtomBytes, sfull);
          }
          ++seg;
        }
      }
      for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait_drain(qfull(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
      if (issued > 0) mbar_wait_drain(doutfull, static_cast<uint32_t>((issued - 1) & 1));
      if (seg > 0) mbar_wait_drain(sfull, static_cast<uint32_t>((seg - 1) & 1));
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, G::kNPad, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc3 = idesc_bf16_f32(128, D, true, true);
      constexpr uint32_t idesc3z = idesc_bf16_f32(128, 16, true, true);
      constexpr int KPA = G::kAtomElems / 16;
      constexpr uint32_t kSAtom = G::kNPad * G::kRowBytes;
      int64_t i = 0, seg = 0;
      for (; cur.valid(); cur.advance(), ++i) {
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        if (cur.first) {
          if (!mbar_wait(sfull, static_cast<uint32_t>(seg & 1), abort, kCode)) break;
        }
        const int s = static_cast<int>(i % S);
        if (!mbar_wait(qrelu(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
        if (!mbar_wait(acc1_free, ph ^ 1u, abort, kCode)) break;
        tc_fence_after();
        // MMA1: [num | den] = phi(Q) . S_f
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int a = kk / KPA, w = kk % KPA;
          const uint64_t ad = smem_desc(q_buf(s) + a * G::kAtomTileBytes + w * 32, 16,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd = smem_desc(s_buf + a * kSAtom + w * 32, 16, G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + C::kAcc1, ad, bd, idesc1, kk > 0 ? 1u : 0u);
        }
        mma_commit(acc1_full);
        // MMA2: dout . S_f[:, :d]^T = dout . S_hi^T + dout . S_lo^T  (K over the
        // d value columns), once dout has landed and the previous tile's result
        // has been read
        if (!mbar_wait(doutfull, ph, abort, kCode)) break;
        if (!mbar_wait(acc2_free, ph ^ 1u, abort, kCode)) break;
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t sb = part == 0 ? s_buf : s_lo;
          const uint32_t lbo = part == 0 ? kSAtom : static_cast<uint32_t>(C::kSLoAtomBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int a = kk / KPA, w = kk % KPA;
            const uint64_t ad = smem_desc(d_buf + a * G::kAtomTileBytes + w * 32, 16,
                                          G::kGroupBytes, G::kLayout);
            const uint64_t bd = smem_desc(sb + kk * 2 * G::kGroupBytes, lbo, G::kGroupBytes,
                                          G::kLayout);
            mma_bf16(tmem + C::kAcc2, ad, bd, idesc2, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(acc2_full);
        // D of this tile (written over dout after MMA2 read it) and, at a
        // unit's start, the free L_f accumulator
        if (!mbar_wait(dfull, ph, abort, kCode)) break;
        if (cur.first &&
            !mbar_wait(acc3_free, static_cast<uint32_t>((seg & 1) ^ 1), abort, kCode))
          break;
        tc_fence_after();
        // MMA3: L_f += phi(Q)^T . D  (K over the tile's tokens): N = d value
        // columns from D_hi's main atoms first, then the release of that
        // buffer (the next dout lands there), then N = 16 from the pad region
        // and D_lo (both written again only after lfree)
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          const uint32_t acc = (cur.first && kk == 0) ? 0u : 1u;
          const uint64_t ad = smem_desc(q_buf(s) + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd = smem_desc(d_buf + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + C::kAcc3, ad, bd, idesc3, acc);
        }
        mma_commit(dfree);
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          const uint32_t acc = (cur.first && kk == 0) ? 0u : 1u;
          const uint64_t ad = smem_desc(q_buf(s) + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bz = smem_desc(d_pad + kk * 512, C::kDPadBytes, 256, kLayoutSW32);
          mma_bf16(tmem + C::kAcc3 + D, ad, bz, idesc3z, acc);
          const uint64_t bl = smem_desc(l_buf + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + C::kAcc3, ad, bl, idesc3, 1u);
        }
        mma_commit(qempty(s));
        mma_commit(lfree);
        if (cur.last) {
          mma_commit(acc3_full);
          mma_commit(sempty);
          ++seg;
        }
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ---------------------------------------------- warps 0-7: ReLU, D, dq, L_f
    // Warps 4-7 apply ReLU one tile ahead, after their part of the previous
    // tile's D (and keep the q > 0 mask); all
    // eight build D, warp w for the token rows of its TMEM lane quarter
    // (w % 4) and the value columns 64 (w / 4) ..; warps 0-3 then form dq and,
    // at a unit's end, write L_f.
    const int q4 = warp & 3;
    const int hc = warp >> 2;        // column half of D
    const int row = q4 * 32 + lane;  // token within the tile (= key feature for L_f)
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    constexpr int CPA = G::kAtomElems / 8;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // S_f[:, d] of the recompute scan
    // ---- ReLU of tile ir (warps 4-7)
    TileCursor cr = cur;
    int64_t ir = 0;
    auto relu = [&]() -> bool {
      constexpr int CPR = G::kChunksPerRow;
      constexpr int RPP = kTileTokens / CPR;
      const int rt = threadIdx.x - 128;
      const int c = rt % CPR;
      const int r0 = rt / CPR;
      const uint32_t off0 =
          (c / CPA) * G::kAtomTileBytes + r0 * G::kRowBytes + G::swz(r0, c % CPA) * 16;
      const int s = static_cast<int>(ir % S);
      const int mr = static_cast<int>(ir % R);
      if (!warp_wait(qfull(s), static_cast<uint32_t>((ir / S) & 1), abort, kCode)) return false;
      if (!warp_wait(maskfree(mr), static_cast<uint32_t>(((ir / R) & 1) ^ 1), abort, kCode))
        return false;
      const uint32_t base = q_buf(s) + off0;
      uint8_t* mrow = mask_ring + mr * C::kMaskBytes;
#pragma unroll
      for (int m = 0; m < CPR; ++m) {
        const uint32_t addr = base + m * RPP * G::kRowBytes;
        uint4 w = ld_shared_v4(addr);
        relu8(w);
        st_shared_v4(addr, w);
        // bit e set <=> feature 8c + e of this token is positive
        uint32_t bits = 0;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bits |= ((ws[e] & 0x7FFFu) != 0u ? 1u : 0u) << (2 * e);
          bits |= ((ws[e] & 0x7FFF0000u) != 0u ? 1u : 0u) << (2 * e + 1);
        }
        mrow[(r0 + m * RPP) * (D / 8) + c] = static_cast<uint8_t>(bits);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(qrelu(s));
        mbar_arrive(maskfull(mr));
      }
      cr.advance();
      ++ir;
      return true;
    };
    bool ok = hc == 0 || !cr.valid() || relu();
    int64_t i = 0, seg = 0;
    int b = 0, f = 0, h = 0;
    for (; ok && cur.valid(); cur.advance(), ++i) {
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
      const int tok = cur.t * kTileTokens + row;
      const bool valid_tok = tok < p.T;
      // ---- Epi1: D = [dout / den | -(dout . num) / den^2] in hi/lo parts,
      // value columns 64 hc .. 64 hc + 63 of this warp's rows
      if (!warp_wait(acc1_full, ph, abort, kCode)) break;
      if (!warp_wait(doutfull, ph, abort, kCode)) break;  // dout in D_hi (previous D read)
      if (!warp_wait(lfree, ph ^ 1u, abort, kCode)) break;  // the previous MMA3 read D_lo
      tc_fence_after();
      const uint32_t t1 = tmem + lane_base + C::kAcc1;
      uint32_t dr;
      tmem_ld_1col(t1 + D, dr);
      tmem_wait_ld();
      const float rden = 1.0f / (__uint_as_float(dr) + p.eps);
      float dot4[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
      uint32_t dhi[D / 4];                   // this half-row of D_hi, written after MMA2
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t r[32];
        tmem_ld_32cols(t1 + hc * 64 + cc * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 8 columns = one 16-byte chunk of D
          const int chunk = hc * 8 + cc * 4 + ch;
          const int a = chunk / CPA, cin = chunk % CPA;
          const uint32_t off = a * G::kAtomTileBytes + row * G::kRowBytes + G::swz(row, cin) * 16;
          const uint4 dq4 = ld_shared_v4(d_buf + off);  // dout (zero past the frame's end)
          const uint32_t dw[4] = {dq4.x, dq4.y, dq4.z, dq4.w};
          uint32_t wl[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const uint32_t wpair = dw[e2];
            const float d0 = bf16lo_to_f32(wpair), d1 = bf16hi_to_f32(wpair);
            dot4[e2] = fmaf(d0, __uint_as_float(r[8 * ch + 2 * e2]), dot4[e2]);
            dot4[e2] = fmaf(d1, __uint_as_float(r[8 * ch + 2 * e2 + 1]), dot4[e2]);
            const float x0 = d0 * rden, x1 = d1 * rden;
            const uint32_t w = pack_bf16x2(x0, x1);
            dhi[(cc * 4 + ch) * 4 + e2] = w;
            wl[e2] = pack_bf16x2(x0 - bf16lo_to_f32(w), x1 - bf16hi_to_f32(w));
          }
          st_shared_v4(l_buf + off, make_uint4(wl[0], wl[1], wl[2], wl[3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc1_free);
      // dout . num: the two column halves meet in shared memory (a buffer per
      // tile parity: a warp writes tile i + 2's only after both arrived for
      // tile i + 1, i.e. after its partner read tile i's)
      float* dx = dot_x + (i & 1) * 2 * kTileTokens;
      dx[hc * kTileTokens + row] = (dot4[0] + dot4[1]) + (dot4[2] + dot4[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar(q4));
      if (!warp_wait(xbar(q4), ph, abort, kCode)) break;
      const float dot = dx[row] + dx[kTileTokens + row];
      const float dden = valid_tok ? -dot * rden * rden : 0.f;
      if (hc == 0) {
        const float dden_lo = dden - bf16lo_to_f32(pack_bf16x2(dden, 0.f));
        // pad region row: chunk 0 (columns 0..7) sits at chunk slot (row >> 2) & 1;
        // column 0 = dden rounded to bf16, column 1 = the rounding's remainder
        const uint32_t poff = row * 32 + ((row >> 2) & 1) * 16;
        st_shared_v4(d_pad + poff, make_uint4(pack_bf16x2(dden, dden_lo), 0u, 0u, 0u));
      }
      // D_hi over dout once MMA2 has read it
      if (!warp_wait(acc2_full, ph, abort, kCode)) break;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const int chunk = hc * 8 + k;
        const int a = chunk / CPA, cin = chunk % CPA;
        const uint32_t off = a * G::kAtomTileBytes + row * G::kRowBytes + G::swz(row, cin) * 16;
        st_shared_v4(d_buf + off, make_uint4(dhi[k * 4], dhi[k * 4 + 1], dhi[k * 4 + 2],
                                             dhi[k * 4 + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(dfull);

      // ---- Epi2: dq = 1[q > 0] * (rden * (dout S^T) + dden * S_f[:, d]),
      // feature columns 64 hc .. 64 hc + 63 of this warp's rows
      tc_fence_after();
      const int mr = static_cast<int>(i % R);
      if (!warp_wait(maskfull(mr), static_cast<uint32_t>((i / R) & 1), abort, kCode)) break;
      const uint2 mk = *reinterpret_cast<const uint2*>(mask_ring + mr * C::kMaskBytes +
                                                       row * (D / 8) + hc * 8);
      __syncwarp();
      if (lane == 0) mbar_arrive(maskfree(mr));
      const uint32_t mwords[2] = {mk.x, mk.y};
      const float4* sd = reinterpret_cast<const float4*>(
          p.states + static_cast<int64_t>(cur.u) * PF + static_cast<int64_t>(D) * D + hc * 64);
      const uint32_t t2 = tmem + lane_base + C::kAcc2 + hc * 64;
      const int tok0 = cur.t * kTileTokens + q4 * 32;
      const uint32_t stg = o_base + warp * C::kRoundBytes;
#pragma unroll
      for (int cc = 0; cc < 64 / C::kRoundCols; ++cc) {
        uint32_t r[32];
        tmem_ld_32cols(t2 + cc * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int col8 = cc * 4 + ch;  // 8-feature chunk of this half
          const uint32_t mb = (mwords[col8 >> 2] >> (8 * (col8 & 3))) & 0xFFu;
          const float4 s0 = __ldg(sd + 2 * col8), s1 = __ldg(sd + 2 * col8 + 1);
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float y = fmaf(rden, __uint_as_float(r[8 * ch + e]), dden * sv[e]);
            x[e] = ((mb >> e) & 1u) != 0u ? y : 0.f;
          }
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) pk[ch * 4 + e2] = pack_bf16x2(x[2 * e2], x[2 * e2 + 1]);
        }
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)  // 64-byte swizzle: chunk ch of row lane
          st_shared_v4(stg + lane * 64 + ((ch ^ ((lane >> 1) & 3)) * 16),
                       make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (tok0 < p.T)
            tma_store_5d(&tm_dq, stg, hc * 64 + cc * C::kRoundCols, h, tok0, f, b);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc2_free);
      if (hc == 1) {
        // the next tile's ReLU after this tile's D and dq: its q lands after
        // this tile's dout, and D is on the tile chain
        if (cr.valid() && !relu()) break;
        continue;
      }
      // ---- Epi3 (unit end): L_f partial, row j = state column, column i = row
      if (cur.last) {
        if (!warp_wait(acc3_full, static_cast<uint32_t>(seg & 1), abort, kCode)) break;
        tc_fence_after();
        float* dst = p.partial + cur.slot() * static_cast<int64_t>(PF) + row;
        const uint32_t t3 = tmem + lane_base + C::kAcc3;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(t3 + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) dst[(cc * 32 + jj) * D] = __uint_as_float(r[jj]);
        }
        uint32_t zr, zl;  // the normaliser column: hi and lo parts of dden
        tmem_ld_1col(t3 + D, zr);
        tmem_ld_1col(t3 + D + 1, zl);
        tmem_wait_ld();
        dst[static_cast<int64_t>(D) * D] = __uint_as_float(zr) + __uint_as_float(zl);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc3_free);
        ++seg;
      }
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
