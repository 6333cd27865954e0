// gla_bwd_q.cuh -- query side of the backward pass on tcgen05.
//
// For the queries of frame f, with S_f the forward prefix state:
//   num_t = phi(q_t) S_f[:, :d],  den_t = phi(q_t) S_f[:, d] + eps,  rden_t = 1 / den_t
//   dnum_t = dout_t rden_t,       dden_t = -(dout_t . num_t) rden_t^2
//   dq_t  = 1[q_t > 0] * (rden_t (dout_t S_f[:, :d]^T) + dden_t S_f[:, d])
//   L_f   = sum_{t in f} phi(q_t)^T [dnum_t | dden_t]     (frame f's state gradient)
// Per 128-token tile, three contractions into TMEM:
//   MMA1  [num | den] = phi(Q) S_f         A = phi(Q) K-major, B = S_hi^T image K-major (N = d+16)
//   MMA2  dout S_f[:, :d]^T                A = dout K-major, B = S_hi^T then S_lo^T MN-major
//   MMA3  L_f[:, :d] += (rden phi(Q))^T dout
//                                          A = (rden phi(Q))^T from TMEM (hi, then lo part),
//                                          B = dout MN-major
// The 1/den scale of dnum is moved from dout onto phi(Q): dnum's
// contraction reads dout exactly as loaded, and the scaled, transposed
// queries go to tensor memory as the A operand, as a hi/lo pair of bf16
// copies (rden phi(q) = hi + lo), in the columns of MMA1's accumulator once
// the epilogue has read it (MMA1 of the next tile is issued after MMA3 has
// completed).  No D tile is built in shared memory, so the dout tile is
// released right after MMA3 and is double-buffered like q.  The normaliser
// column of L_f (sum_t phi(q_t) dden_t) is formed in fp32 on the CUDA cores
// on the way; dq is formed
// from dout itself against the hi/lo pair of bf16 copies of S_f with the
// 1/den scale and the normaliser term added in fp32.  In a frame of few
// tokens the two terms of dq cancel almost exactly (out_t stays near v_t),
// and the gate gradient <G_f, S_{f-1}> and dk sum thousands of products of
// L_f with random signs: one bf16 rounding of either operand in these
// contractions would leave residue near the tolerance, hence the pairs.
// L_f is accumulated over a unit's tiles and written as an fp32 partial in
// the forward increment's slot layout (row d = the normaliser column) for
// the reverse scan.
// Warp roles: 0-7 epilogue (warp w: TMEM lane quarter w % 4, column half
// w / 4): the rden/dden exchange, the A operand (key features = lanes,
// tokens 64 (w / 4) .. of the tile), ReLU of the next tile, dq, L_f;
// 8 TMA; 9 MMA.
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"  // warp_wait, unit_coords, IncCfg
#include "sm100_ptx.cuh"

namespace gla {

template <int D>
struct BwdQCfg {
  using G = Geo<D>;
  static_assert(D == 128, "the backward kernels are built for d = 128");
  static constexpr int kStages = 2;                             // q and dout tiles
  static constexpr int kSHiAtomBytes = G::kNPad * G::kRowBytes;  // image atom + zero rows
  static constexpr int kSHiBytes = G::kAtoms * kSHiAtomBytes;    // S_f^T image (hi)
  static constexpr int kSLoAtomBytes = D * G::kRowBytes;         // value rows of one atom
  static constexpr int kSLoBytes = G::kAtoms * kSLoAtomBytes;    // S_f^T image (lo)
  // dq stores: rounds of 32 tokens x 32 features per warp (64-byte swizzle,
  // 2 KB), one buffer for each of the eight warps
  static constexpr int kRoundCols = 32;
  static constexpr int kRoundBytes = 32 * kRoundCols * 2;
  static constexpr int kStageOutBytes = 8 * kRoundBytes;
  static constexpr int kMaskRing = 2;
  static constexpr int kMaskBytes = kTileTokens * (D / 8);      // one bit per feature
  static constexpr int kAcc1 = 0;    // [num | den]   : N = d + 16
  static constexpr int kAHi = 0;     // (rden phi(Q))^T, hi part: 64 columns of bf16 pairs
  static constexpr int kALo = 64;    // its lo part (both over num once it is read)
  static constexpr int kAcc2 = 160;  // dout S^T      : N = d
  static constexpr int kAcc3 = 288;  // L_f[:, :d]    : N = d
  static constexpr int kTmemCols = 512;
  static constexpr int kThreads = 320;
  static constexpr int kBarCount = 5 * kStages + 12 + 8 + 2 * kMaskRing;
  // per tile parity: [column half][token] dot partial sums; [token] rden and
  // dden
  static constexpr int kXchgBytes = 2 * 2 * kTileTokens * 4;
  static constexpr int kRdBytes = 2 * 2 * kTileTokens * 4;
  static constexpr int kZBytes = 2 * D * 4;    // S_f[:, d] in fp32, per unit parity
  static constexpr int kNxBytes = D * 4;       // normaliser exchange at a unit's end
  static constexpr int kSmemBytes = 1024 + 2 * kStages * G::kTileBytes + kSHiBytes + kSLoBytes +
                                    kStageOutBytes + kMaskRing * kMaskBytes + kXchgBytes +
                                    kRdBytes + kZBytes + kNxBytes + kBarCount * 8 + 16;
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

// Bit e set <=> bf16 element e of the eight in x (all >= +-0 after ReLU) is
// nonzero: per 16-bit half, (h & 0x7FFF) + 0x7FFF carries into bit 15 iff
// h & 0x7FFF != 0, without a carry out of the half; a byte permute gathers
// the four flag bytes of two words and a multiply packs their top bits.
__device__ __forceinline__ uint32_t positive_mask8(const uint4& x) {
  const uint32_t t0 = ((x.x & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x80008000u;
  const uint32_t t1 = ((x.y & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x80008000u;
  const uint32_t t2 = ((x.z & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x80008000u;
  const uint32_t t3 = ((x.w & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x80008000u;
  // bytes [w.lo flag, w.hi flag, w'.lo flag, w'.hi flag], each 0x80 or 0
  const uint32_t u = __byte_perm(t0, t1, 0x7531) >> 7;
  const uint32_t v = __byte_perm(t2, t3, 0x7531) >> 7;
  // byte k (0 or 1) of u lands on bit 24 + k of u * 0x01020408, no carries
  const uint32_t lo = (u * 0x01020408u) >> 24;
  const uint32_t hi = (v * 0x01020408u) >> 24;
  return (lo & 0xFu) | ((hi & 0xFu) << 4);
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    gla_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_dout,
                     const __grid_constant__ CUtensorMap tm_dq, const BwdQParams p) {
  using G = Geo<D>;
  using C = BwdQCfg<D>;
  constexpr int S = C::kStages;
  constexpr int R = C::kMaskRing;
  constexpr unsigned kCode = 32u;
  constexpr int PF = IncCfg<D>::kPartialFloats;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto q_buf = [&](int s) { return sbase + s * G::kTileBytes; };
  auto d_buf = [&](int s) { return sbase + (S + s) * G::kTileBytes; };
  const uint32_t s_hi = sbase + 2 * S * G::kTileBytes;
  const uint32_t s_lo = s_hi + C::kSHiBytes;
  const uint32_t o_base = s_lo + C::kSLoBytes;  // dq staging: one round per warp
  const uint32_t mask_base = o_base + C::kStageOutBytes;
  const uint32_t xchg = mask_base + R * C::kMaskBytes;  // float [parity][half][token]
  const uint32_t rd = xchg + C::kXchgBytes;             // float [parity][rden | dden][token]
  const uint32_t zb = rd + C::kRdBytes;                 // float [unit parity][d]
  const uint32_t nx = zb + C::kZBytes;                  // float [d]
  uint8_t* mask_ring = smem + (mask_base - sbase);
  float* xchg_p = reinterpret_cast<float*>(smem + (xchg - sbase));
  float* rd_p = reinterpret_cast<float*>(smem + (rd - sbase));
  float* nx_p = reinterpret_cast<float*>(smem + (nx - sbase));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (nx + C::kNxBytes - sbase));
  const uint32_t bar0 = smem_u32(bars);
  auto qfull = [&](int s) { return bar0 + 8u * s; };
  auto qrelu = [&](int s) { return bar0 + 8u * (S + s); };
  auto qempty = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto dfull = [&](int s) { return bar0 + 8u * (3 * S + s); };
  auto dempty = [&](int s) { return bar0 + 8u * (4 * S + s); };
  const uint32_t sfull = bar0 + 8u * (5 * S + 0);
  const uint32_t sempty = bar0 + 8u * (5 * S + 1);
  const uint32_t acc1_full = bar0 + 8u * (5 * S + 2);
  const uint32_t acc1_free = bar0 + 8u * (5 * S + 3);
  const uint32_t acc2_full = bar0 + 8u * (5 * S + 4);
  const uint32_t acc2_free = bar0 + 8u * (5 * S + 5);
  const uint32_t afull = bar0 + 8u * (5 * S + 6);    // A operand written
  const uint32_t afree = bar0 + 8u * (5 * S + 7);    // MMA3 read it
  const uint32_t acc3_full = bar0 + 8u * (5 * S + 8);
  const uint32_t acc3_free = bar0 + 8u * (5 * S + 9);
  const uint32_t rdfull = bar0 + 8u * (5 * S + 10);  // rden, dden of every token written
  const uint32_t done_bar = bar0 + 8u * (5 * S + 11);
  // both column halves of lane quarter q wrote their partial sums
  auto xbar = [&](int q) { return bar0 + 8u * (5 * S + 12 + q); };
  // column half 1 of lane quarter q wrote its normaliser sums
  auto nbar = [&](int q) { return bar0 + 8u * (5 * S + 16 + q); };
  auto maskfull = [&](int m) { return bar0 + 8u * (5 * S + 20 + m); };
  auto maskfree = [&](int m) { return bar0 + 8u * (5 * S + 20 + R + m); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  TileCursor cur;
  cur.init(p.wp, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(qfull(s), 1);
      mbar_init(qrelu(s), 8);
      mbar_init(qempty(s), 8);
      mbar_init(dfull(s), 1);
      mbar_init(dempty(s), 1);
    }
    for (int m = 0; m < R; ++m) {
      mbar_init(maskfull(m), 8);
      mbar_init(maskfree(m), 8);
    }
    mbar_init(sfull, 1);
    mbar_init(sempty, 1);
    mbar_init(acc1_full, 1);
    mbar_init(acc1_free, 8);
    mbar_init(acc2_full, 1);
    mbar_init(acc2_free, 8);
    mbar_init(afull, 8);
    mbar_init(afree, 1);
    mbar_init(acc3_full, 1);
    mbar_init(acc3_free, 8);
    mbar_init(rdfull, 4);
    mbar_init(done_bar, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(xbar(q), 2);
      mbar_init(nbar(q), 1);
    }
    *abort = 0;
    fence_mbar_init();
  }
  {
    // zero: the S_hi image's padding rows (the loads write rows 0 .. d only)
    constexpr int kPadRows = G::kNPad - G::kStateRows;
    constexpr int kPadChunks = G::kAtoms * kPadRows * (G::kRowBytes / 16);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = threadIdx.x; idx < kPadChunks; idx += C::kThreads) {
      const int ch = idx % (G::kRowBytes / 16);
      const int rr = (idx / (G::kRowBytes / 16)) % kPadRows;
      const int at = idx / ((G::kRowBytes / 16) * kPadRows);
      st_shared_v4(s_hi + at * C::kSHiAtomBytes + (G::kStateRows + rr) * G::kRowBytes + ch * 16, z);
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

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_dout);
      asm volatile("griddepcontrol.wait;" ::: "memory");  // S images of the forward recompute
      int64_t nq = 0, nd = 0, seg = 0;
      int b = 0, f = 0, h = 0;
      for (; cur.valid(); cur.advance()) {
        if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
        // q once the ReLU warps have read the stage's previous tile for the
        // last time (its A operand written), dout once MMA3 has read it,
        // then (at a unit's start) the state images once the previous unit's
        // last MMA3 has run
        const int sq = static_cast<int>(nq % S);
        if (!mbar_wait(qempty(sq), static_cast<uint32_t>(((nq / S) & 1) ^ 1), abort, kCode))
          break;
        mbar_arrive_expect_tx(qfull(sq), G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(q_buf(sq) + a * G::kAtomTileBytes, &tm_q, qfull(sq), a * G::kAtomElems, h,
                      cur.t * kTileTokens, f, b);
        ++nq;
        const int sd = static_cast<int>(nd % S);
        if (!mbar_wait(dempty(sd), static_cast<uint32_t>(((nd / S) & 1) ^ 1), abort, kCode))
          break;
        mbar_arrive_expect_tx(dfull(sd), G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(d_buf(sd) + a * G::kAtomTileBytes, &tm_dout, dfull(sd), a * G::kAtomElems,
                      h, cur.t * kTileTokens, f, b);
        ++nd;
        if (cur.first) {
          if (!mbar_wait(sempty, static_cast<uint32_t>((seg & 1) ^ 1), abort, kCode)) break;
          mbar_arrive_expect_tx(sfull, G::kImageBytes + C::kSLoBytes + D * 4);
          const int64_t off = static_cast<int64_t>(cur.u) * G::kImageBytes;
#pragma unroll
          for (int a = 0; a < G::kAtoms; ++a) {
            bulk_load(s_hi + a * C::kSHiAtomBytes, p.image + off + a * G::kImageAtomBytes,
                      G::kImageAtomBytes, sfull);
            bulk_load(s_lo + a * C::kSLoAtomBytes, p.image_lo + off + a * G::kImageAtomBytes,
                      C::kSLoAtomBytes, sfull);
          }
          bulk_load(zb + (seg & 1) * D * 4,
                    p.states + static_cast<int64_t>(cur.u) * PF + static_cast<int64_t>(D) * D,
                    D * 4, sfull);
          ++seg;
        }
      }
      // let every copy in flight land before the CTA exits
      for (int64_t i = (nq > S ? nq - S : 0); i < nq; ++i)
        mbar_wait_drain(qfull(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
      for (int64_t i = (nd > S ? nd - S : 0); i < nd; ++i)
        mbar_wait_drain(dfull(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
      if (seg > 0) mbar_wait_drain(sfull, static_cast<uint32_t>((seg - 1) & 1));
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, G::kNPad, false, false);
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc3 = idesc_bf16_f32(128, D, false, true);
      constexpr int KPA = G::kAtomElems / 16;
      int64_t seg1 = 0, seg3 = 0;
      // MMA1 of tile k: [num | den] = phi(Q) . S_f
      auto mma1 = [&](const TileCursor& c, int64_t k) -> bool {
        const int s = static_cast<int>(k % S);
        if (c.first) {
          if (!mbar_wait(sfull, static_cast<uint32_t>(seg1 & 1), abort, kCode)) return false;
          ++seg1;
        }
        if (!mbar_wait(qrelu(s), static_cast<uint32_t>((k / S) & 1), abort, kCode)) return false;
        if (!mbar_wait(acc1_free, static_cast<uint32_t>((k & 1) ^ 1), abort, kCode)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int a = kk / KPA, w = kk % KPA;
          const uint64_t ad = smem_desc(q_buf(s) + a * G::kAtomTileBytes + w * 32, 16,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd =
              smem_desc(s_hi + a * C::kSHiAtomBytes + w * 32, 16, G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + C::kAcc1, ad, bd, idesc1, kk > 0 ? 1u : 0u);
        }
        mma_commit(acc1_full);
        return true;
      };
      // MMA2 of tile k: dout . S_f[:, :d]^T = dout . S_hi^T + dout . S_lo^T
      // (K over the d value columns)
      auto mma2 = [&](int64_t k) -> bool {
        const int s = static_cast<int>(k % S);
        if (!mbar_wait(dfull(s), static_cast<uint32_t>((k / S) & 1), abort, kCode)) return false;
        if (!mbar_wait(acc2_free, static_cast<uint32_t>((k & 1) ^ 1), abort, kCode)) return false;
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t sb = part == 0 ? s_hi : s_lo;
          const uint32_t lbo = part == 0 ? C::kSHiAtomBytes : C::kSLoAtomBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int a = kk / KPA, w = kk % KPA;
            const uint64_t ad = smem_desc(d_buf(s) + a * G::kAtomTileBytes + w * 32, 16,
                                          G::kGroupBytes, G::kLayout);
            const uint64_t bd = smem_desc(sb + kk * 2 * G::kGroupBytes, lbo, G::kGroupBytes,
                                          G::kLayout);
            mma_bf16(tmem + C::kAcc2, ad, bd, idesc2, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(acc2_full);
        return true;
      };
      // MMA3 of tile k: L_f[:, :d] += (rden phi(Q))^T_hi . dout + (..)^T_lo . dout
      // (K over the tile's tokens)
      auto mma3 = [&](const TileCursor& c, int64_t k) -> bool {
        const int s = static_cast<int>(k % S);
        if (!mbar_wait(afull, static_cast<uint32_t>(k & 1), abort, kCode)) return false;
        if (c.first &&
            !mbar_wait(acc3_free, static_cast<uint32_t>((seg3 & 1) ^ 1), abort, kCode))
          return false;
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t at = tmem + (part == 0 ? C::kAHi : C::kALo);
#pragma unroll
          for (int kk = 0; kk < kTileTokens / 16; ++kk) {
            const uint64_t bd = smem_desc(d_buf(s) + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                          G::kGroupBytes, G::kLayout);
            mma_bf16_ts(tmem + C::kAcc3, at + kk * 8, bd, idesc3,
                        (c.first && part == 0 && kk == 0) ? 0u : 1u);
          }
        }
        mma_commit(afree);
        mma_commit(dempty(s));
        if (c.last) {
          mma_commit(acc3_full);
          mma_commit(sempty);  // MMA1 and MMA2 of the unit's last tile were issued before
          ++seg3;
        }
        return true;
      };
      // Order: this tile's MMA3, then MMA1 and MMA2 of the next tile (its q
      // is ReLU'd after this tile's A operand is written); MMA1 writes the
      // columns MMA3 reads A from, so it waits for MMA3 to complete
      bool ok = !cur.valid() || (mma1(cur, 0) && mma2(0));
      for (int64_t i = 0; ok && cur.valid(); cur.advance(), ++i) {
        TileCursor nx = cur;
        nx.advance();
        if (!mma3(cur, i)) break;
        if (!nx.valid()) continue;
        if (!mbar_wait(afree, static_cast<uint32_t>(i & 1), abort, kCode)) break;
        if (!(mma1(nx, i + 1) && mma2(i + 1))) break;
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // ------------------------------------- warps 0-7: ReLU, rden/dden, A, dq, L_f
    const int q4 = warp & 3;
    const int hc = warp >> 2;        // column half / token half
    const int row = q4 * 32 + lane;  // token of the tile (Epi1, dq); key feature (A, L_f)
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    constexpr int CPA = G::kAtomElems / 8;
    asm volatile("griddepcontrol.wait;" ::: "memory");  // partial slots of the forward
    // ---- ReLU of tile ir in place, with the q > 0 mask for dq
    TileCursor cr = cur;
    int64_t ir = 0;
    auto relu = [&]() -> bool {
      constexpr int CPR = G::kChunksPerRow;
      constexpr int RPP = 256 / CPR;
      const int c = threadIdx.x % CPR;
      const int r0 = threadIdx.x / CPR;
      const uint32_t off0 =
          (c / CPA) * G::kAtomTileBytes + r0 * G::kRowBytes + G::swz(r0, c % CPA) * 16;
      const int s = static_cast<int>(ir % S);
      const int mr = static_cast<int>(ir % R);
      if (!warp_wait_fast(qfull(s), static_cast<uint32_t>((ir / S) & 1), abort, kCode)) return false;
      if (!warp_wait_fast(maskfree(mr), static_cast<uint32_t>(((ir / R) & 1) ^ 1), abort, kCode))
        return false;
      uint4* qv = reinterpret_cast<uint4*>(smem + (q_buf(s) - sbase) + off0);
      uint8_t* mrow = mask_ring + mr * C::kMaskBytes + r0 * (D / 8) + c;
      constexpr int kPass = kTileTokens / RPP;
      constexpr int kStep = RPP * G::kRowBytes / 16;  // uint4 per pass
      uint4 w[kPass];
#pragma unroll
      for (int m = 0; m < kPass; ++m) w[m] = qv[m * kStep];
#pragma unroll
      for (int m = 0; m < kPass; ++m) {
        relu8(w[m]);
        qv[m * kStep] = w[m];
        mrow[m * RPP * (D / 8)] = positive_mask8(w[m]);
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
    bool ok = !cr.valid() || relu();
    int64_t i = 0, useg = -1;
    int b = 0, f = 0, h = 0;
    // sums over this warp's tokens of phi(q_t)[j] dden_t, per unit, for the
    // key features j = 32 q4 + 16 lb + 8 fh + lane / 4 (index 2 lb + fh), each
    // over this thread's token pairs
    float nq[4] = {0.f, 0.f, 0.f, 0.f};
    for (; ok && cur.valid(); cur.advance(), ++i) {
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const int s = static_cast<int>(i % S);
      const uint32_t sph = static_cast<uint32_t>((i / S) & 1);
      if (cur.first) {
        unit_coords(cur.u, p.H, p.F, b, f, h);
        ++useg;
        if (!warp_wait_fast(sfull, static_cast<uint32_t>(useg & 1), abort, kCode)) break;  // z
      }
      const float* zrow = reinterpret_cast<const float*>(smem + (zb - sbase)) + (useg & 1) * D;
      const int tok = cur.t * kTileTokens + row;
      const bool valid_tok = tok < p.T;
      // ---- Epi1: den, and the half-row partial sum dout . num (value columns
      // 64 hc ..) of this warp's tokens
      if (!warp_wait_fast(acc1_full, ph, abort, kCode)) break;
      if (!warp_wait_fast(dfull(s), sph, abort, kCode)) break;
      if (!warp_wait_fast(qrelu(s), sph, abort, kCode)) break;
      tc_fence_after();
      float dot4[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
      float rden;
      {
        uint32_t dr;
        tmem_ld_1col(tmem + lane_base + C::kAcc1 + D, dr);
        const uint32_t t1 = tmem + lane_base + C::kAcc1 + hc * 64;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(t1 + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {  // 8 columns = one 16-byte chunk
            const int cin = (cc * 4 + ch) % CPA;
            const uint32_t off = hc * G::kAtomTileBytes + row * G::kRowBytes + G::swz(row, cin) * 16;
            const uint4 d4 = *reinterpret_cast<const uint4*>(smem + (d_buf(s) - sbase) + off);
            const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              dot4[e2] = fmaf(bf16lo_to_f32(dw[e2]), __uint_as_float(r[8 * ch + 2 * e2]), dot4[e2]);
              dot4[e2] =
                  fmaf(bf16hi_to_f32(dw[e2]), __uint_as_float(r[8 * ch + 2 * e2 + 1]), dot4[e2]);
            }
          }
        }
        rden = 1.0f / (__uint_as_float(dr) + p.eps);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc1_free);
      }
      // the two column halves meet in shared memory (a buffer per tile
      // parity: a warp writes tile i + 2's only after every warp finished
      // tile i + 1's Epi1, i.e. after its partner read tile i's)
      float* xp = xchg_p + (i & 1) * 2 * kTileTokens;
      xp[hc * kTileTokens + row] = (dot4[0] + dot4[1]) + (dot4[2] + dot4[3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar(q4));
      if (!warp_wait_fast(xbar(q4), ph, abort, kCode)) break;
      const float dot = xp[row] + xp[kTileTokens + row];
      const float dden = valid_tok ? -dot * rden * rden : 0.f;
      float* rdp = rd_p + (i & 1) * 2 * kTileTokens;
      if (hc == 0) {
        rdp[row] = rden;
        rdp[kTileTokens + row] = dden;
        __syncwarp();
        if (lane == 0) mbar_arrive(rdfull);
      }
      // ---- A operand: lanes = key features, columns = token pairs;
      // A[j][t] = rden_t phi(q_t)[j] as hi + lo, tokens 64 hc .. 64 hc + 63;
      // the normaliser column of L_f in fp32 on the way
      if (!warp_wait_fast(rdfull, ph, abort, kCode)) break;
      if (!warp_wait_fast(afree, ph ^ 1u, abort, kCode)) break;
      tc_fence_after();
      {
        // 8 x 8 blocks of phi(Q) (token rows) read transposed: thread t gets,
        // per block, one key feature (t / 4 of the block's 8) at the token
        // pair 2 (t % 4), 2 (t % 4) + 1, which is the 16-lane TMEM store's
        // layout (lanes = key features, columns = token pairs)
        const float* rdn = rd_p + (i & 1) * 2 * kTileTokens + hc * 64;
        const float* ddn = rdn + kTileTokens;
        const int mi = lane >> 3;                       // this lane's ldmatrix block
        const int tp = 2 * (lane & 3);                  // first token of this thread's pairs
#pragma unroll
        for (int lb = 0; lb < 2; ++lb) {                // key features 32 q4 + 16 lb ..
          const int fc = q4 * 4 + lb * 2 + (mi & 1);    // 16-byte feature chunk of the row
          const uint32_t fbase = q_buf(s) + (fc / CPA) * G::kAtomTileBytes;
          uint32_t hi[16], lo[16];
          uint64_t na2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int tg = 0; tg < 4; ++tg) {              // tokens 64 hc + 16 tg ..
            const int tr = hc * 64 + tg * 16 + (mi >> 1) * 8 + (lane & 7);
            uint32_t m4[4];
            ldmatrix_x4_trans(fbase + tr * G::kRowBytes + G::swz(tr, fc % CPA) * 16, m4);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {           // token pair tg * 16 + tp + 8 tt
              const int t = tg * 16 + tp + 8 * tt;
              const float2 r2 = *reinterpret_cast<const float2*>(rdn + t);
              const float2 g2 = *reinterpret_cast<const float2*>(ddn + t);
              const uint64_t rr2 = f2_pack(r2.x, r2.y), gg2 = f2_pack(g2.x, g2.y);
#pragma unroll
              for (int fh = 0; fh < 2; ++fh) {         // key feature 16 lb + 8 fh + lane / 4
                const uint32_t pw = m4[2 * tt + fh];
                const uint64_t p2 = f2_pack(bf16lo_to_f32(pw), bf16hi_to_f32(pw));
                float x0, x1;
                f2_unpack(f2_mul(rr2, p2), x0, x1);
                const uint32_t w = pack_bf16x2(x0, x1);
                float l0, l1;
                f2_unpack(f2_sub(f2_pack(x0, x1), f2_pack(bf16lo_to_f32(w), bf16hi_to_f32(w))),
                          l0, l1);
                hi[2 * (2 * tg + tt) + fh] = w;
                lo[2 * (2 * tg + tt) + fh] = pack_bf16x2(l0, l1);
                na2[fh] = f2_fma(p2, gg2, na2[fh]);
              }
            }
          }
          const uint32_t ta = tmem + lane_base + (static_cast<uint32_t>(lb * 16) << 16) + hc * 32;
          tmem_st_16x128b_x8(ta + C::kAHi, hi);
          tmem_st_16x128b_x8(ta + C::kALo, lo);
#pragma unroll
          for (int fh = 0; fh < 2; ++fh) {
            float na0, na1;
            f2_unpack(na2[fh], na0, na1);
            nq[2 * lb + fh] += na0 + na1;
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(afull);
        mbar_arrive(qempty(s));  // q of this tile read for the last time
      }
      // ---- ReLU of the next tile: its load was issued when the tile before
      // this one released its q stage; MMA1 of it runs beside dq
      if (cr.valid() && !relu()) break;

      // ---- Epi2: dq = 1[q > 0] * (rden * (dout S^T) + dden * S_f[:, d]),
      // feature columns 64 hc .. 64 hc + 63 of this warp's tokens
      if (!warp_wait_fast(acc2_full, ph, abort, kCode)) break;
      tc_fence_after();
      const int mr = static_cast<int>(i % R);
      if (!warp_wait_fast(maskfull(mr), static_cast<uint32_t>((i / R) & 1), abort, kCode)) break;
      const uint2 mk = *reinterpret_cast<const uint2*>(mask_ring + mr * C::kMaskBytes +
                                                       row * (D / 8) + hc * 8);
      __syncwarp();
      if (lane == 0) mbar_arrive(maskfree(mr));
      const uint32_t mwords[2] = {mk.x, mk.y};
      const uint32_t t2 = tmem + lane_base + C::kAcc2 + hc * 64;
      const uint64_t rden2 = f2_pack(rden, rden), dden2 = f2_pack(dden, dden);
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
          const float4 s0 = *reinterpret_cast<const float4*>(zrow + hc * 64 + col8 * 8);
          const float4 s1 = *reinterpret_cast<const float4*>(zrow + hc * 64 + col8 * 8 + 4);
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float y0, y1;
            f2_unpack(f2_fma(rden2, f2_pack(__uint_as_float(r[8 * ch + e]),
                                            __uint_as_float(r[8 * ch + e + 1])),
                             f2_mul(dden2, f2_pack(sv[e], sv[e + 1]))),
                      y0, y1);
            x[e] = ((mb >> e) & 1u) != 0u ? y0 : 0.f;
            x[e + 1] = ((mb >> (e + 1)) & 1u) != 0u ? y1 : 0.f;
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

      // ---- Epi3 (unit end): L_f partial, row j = state column, column i =
      // key feature; this warp's lanes, value columns 64 hc ..
      if (cur.last) {
        if (!warp_wait_fast(acc3_full, static_cast<uint32_t>(useg & 1), abort, kCode)) break;
        tc_fence_after();
        float* dst = p.partial + cur.slot() * static_cast<int64_t>(PF) + row;
        const uint32_t t3 = tmem + lane_base + C::kAcc3 + hc * 64;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(t3 + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) dst[(hc * 64 + cc * 32 + jj) * D] = __uint_as_float(r[jj]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc3_free);
        // row d: the two token halves' sums of phi(q_t) dden_t; this warp's
        // share of lane `row`: the four token-pair partials of its quad
        float nacc;
        {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            nq[k] += __shfl_xor_sync(0xffffffffu, nq[k], 1);
            nq[k] += __shfl_xor_sync(0xffffffffu, nq[k], 2);
          }
          const int src = 4 * (lane & 7);               // a thread of feature lane's quad
          const int kk = 2 * (lane >> 4) + ((lane >> 3) & 1);
          float v[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) v[k] = __shfl_sync(0xffffffffu, nq[k], src);
          nacc = kk == 0 ? v[0] : kk == 1 ? v[1] : kk == 2 ? v[2] : v[3];
        }
        if (hc == 1) {
          nx_p[row] = nacc;
          __syncwarp();
          if (lane == 0) mbar_arrive(nbar(q4));
        } else {
          if (!warp_wait_fast(nbar(q4), static_cast<uint32_t>(useg & 1), abort, kCode)) break;
          dst[static_cast<int64_t>(D) * D] = nacc + nx_p[row];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) nq[k] = 0.f;
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
