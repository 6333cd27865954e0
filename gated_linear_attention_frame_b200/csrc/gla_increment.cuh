// gla_increment.cuh -- per-frame state increment on tcgen05 tensor cores.
//
// For every unit u = (b, f, h) it forms dS_f = phi(K_f)^T [V_f | 1], the
// block's own key-value contribution that the SANA-Video talk (block KV cache
// segment) adds to the cached state, as a bf16 x bf16 -> fp32 contraction
// over the frame's tokens:
//   A = phi(K_f)^T  [M = 128 key features (rows >= d are zero), K = tokens]
//   B = V_f         [N = d value features,                     K = tokens]
// Both operands are MN-major in memory (token rows of d contiguous features),
// loaded by TMA in 128-token tiles with 128-byte (64-byte for d = 32)
// swizzle; ReLU is applied in shared memory between the TMA landing and the
// MMA, and the same pass sums phi(K) over tokens for the normaliser column.
//
// Work split: the token tiles of all units go to the persistent CTAs as the
// WorkPlan describes (whole units in full rounds, then a contiguous split of
// the remainder).  A CTA accumulates the tiles of one unit in TMEM and, when
// the unit or its share of it ends, writes an fp32 partial [d + 1][d]
// (transposed: row j = value column, column i = key feature; row d = the
// normaliser column, the four ReLU warps' sums added in a fixed order) to the
// plan's slot.  The scan kernel sums a unit's partials.
//
// Warp roles: warps 0-3 drain TMEM (epilogue), the next kReluWarps (4; 8 in
// the rotary variant, which has more to do per element) apply ReLU, then one
// warp issues TMA and one issues MMAs.
#pragma once

#include "gla_common.cuh"
#include "gla_rope.cuh"
#include "sm100_ptx.cuh"

namespace gla {

template <int D, bool kRope = false, bool kGram = false>
struct IncCfg {
  using G = Geo<D>;
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kAAtoms = 128 / G::kAtomElems;           // A spans M = 128 rows
  static constexpr int kABytes = kAAtoms * G::kAtomTileBytes;   // 32 KB
  static constexpr int kVBytes = G::kTileBytes;
  static constexpr int kStageBytes = kABytes + kVBytes;
  // two buffers of [dS (N = D) | M (N = D, Gram variant)] fp32 accumulators
  static constexpr int kAccCols = kGram ? 2 * D : D;
  static constexpr int kTmemCols = 2 * kAccCols;
  static constexpr int kPartialRows = D + 1;
  static constexpr int kPartialFloats = kPartialRows * D;
  static constexpr int kReluWarps = kRope ? 8 : 4;
  static constexpr int kThreads = (kReluWarps + 6) * 32;        // + epilogue, TMA, MMA warps
  static constexpr int kBarBytes = (3 * kStages + 7) * 8;
  static constexpr int kZBytes = kReluWarps * D * 4;  // per-ReLU-warp normaliser sums
  // single-frame fold (plain layer): a 32 x 33 fp32 transpose tile per epilogue warp
  static constexpr int kFoldBytes = (!kRope && !kGram) ? 4 * 32 * 33 * 4 : 0;
  static constexpr int kSmemBytes =
      1024 + kStages * kStageBytes + kZBytes + kFoldBytes + kBarBytes + 16;
};

// The delta-rule variant at d = 128 hands M_f to the tensor-core scan as
// that scan's A operand: two bf16 images of [D rows i][D elements k] (hi,
// then lo = bf16(M - hi), so that hi + lo carries ~16 bits of M), K-major
// without swizzle: 8-row x 16-byte core matrices, the 16 bytes holding
// elements 8 ch .. 8 ch + 7 of row i at ch * 16 D + 16 i.  Core matrices are
// 128 bytes apart along M and 16 D bytes apart along K, and a warp that owns
// 32 consecutive rows writes one chunk of each as 512 contiguous bytes.
template <int D>
struct GramImage {
  static constexpr int kBytes = D * D * 2;  // one image
  static constexpr int kChunkStride = 16 * D;  // between K chunks (core matrices along K)
  static constexpr int kGroupStride = 128;     // between 8-row groups (along M)
  __host__ __device__ static constexpr int offset(int i, int ch) { return ch * kChunkStride + i * 16; }
};

// hi / lo bf16 split of 8 consecutive fp32 values (x = hi + lo + O(2^-16 |x|))
__device__ __forceinline__ void split_bf16x8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e2 = 0; e2 < 4; ++e2) {
    h[e2] = pack_bf16x2(x[2 * e2], x[2 * e2 + 1]);
    l[e2] = pack_bf16x2(x[2 * e2] - bf16lo_to_f32(h[e2]), x[2 * e2 + 1] - bf16hi_to_f32(h[e2]));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

struct IncParams {
  float* partial;   // [(units + gridDim.x) slots][d + 1][d] fp32
  WorkPlan wp;      // tile assignment (gridDim.x == wp.G)
  int H, F;         // heads, frames
  int T;            // tokens per frame (rotary variant)
  RopeGeo rope;     // rotary variant only
  float* mpartial;  // Gram variant: [(units + gridDim.x) slots][d][d] fp32 partials of
                    // M_f = phi(K_f)^T phi(K_f), rows as the increment partials; at
                    // d = 128 a unit owned whole by one CTA gets the GramImage pair
                    // (hi | lo, d * d * 4 bytes) in its slot instead
  // Single-frame calls of the plain layer (fold = 1): for a unit owned whole
  // by one CTA the scan's step S = a S_in + dS is done here, from TMEM, at the
  // unit's end (overlapping the CTA's next tiles); a unit whose tiles are
  // split over several CTAs writes its partials as usual, and the scan runs
  // over those units alone.
  int fold;
  const float* gate;        // [B, 1, H] gate logits
  const float* state_in;    // [B, H, d, d+1] or nullptr (zero state)
  float* state_out;         // [B, H, d, d+1] or nullptr (not written; may alias state_in)
  uint8_t* image;           // [units][kImageBytes] bf16 S^T images for the output kernel
};

// (b, f, h) of unit u = (b * F + f) * H + h.
__device__ __forceinline__ void unit_coords(int32_t u, int H, int F, int& b, int& f, int& h) {
  h = u % H;
  const int32_t bf = u / H;
  f = bf % F;
  b = bf / F;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          unsigned int code) {
  const int lane = threadIdx.x & 31;
  int ok = 0;
  if (lane == 0) ok = mbar_wait(bar, parity, abort, code) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_try_wait(bar, parity);  // completed phase: acquire for every lane
  return ok != 0;
}

// A wait on a phase that has most likely completed already: one vote of the
// warp on a non-blocking test, the bounded warp_wait otherwise.
__device__ __forceinline__ bool warp_wait_fast(uint32_t bar, uint32_t parity, volatile int* abort,
                                               unsigned int code) {
  if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
  return warp_wait(bar, parity, abort, code);
}

// kRope: the rotary variant (gla_rope.cuh): phi(K) is rotated in shared
// memory after its normaliser sums are taken, so the contraction forms
// (R phi(K))^T V while row d keeps sum phi(k).
// kGram: the delta-rule variant also forms M_f = phi(K_f)^T phi(K_f) from the
// same shared-memory tile (B = phi(K) read MN-major like A), a second
// accumulator beside dS_f, written as a second fp32 partial.
template <int D, bool kRope = false, bool kGram = false>
__global__ void __launch_bounds__(IncCfg<D, kRope, kGram>::kThreads, 1)
    gla_increment_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const IncParams p) {
  using G = Geo<D>;
  static_assert(!(kRope && kGram), "one variant at a time");
  using C = IncCfg<D, kRope, kGram>;
  constexpr int AC = C::kAccCols;
  constexpr int RW = C::kReluWarps;
  constexpr int kTmaWarp = 4 + RW, kMmaWarp = 5 + RW;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 1u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* zpart = reinterpret_cast<float*>(smem + S * C::kStageBytes);  // [RW][D]
  float* fold_t = reinterpret_cast<float*>(smem + S * C::kStageBytes + C::kZBytes);  // [4][32][33]
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kZBytes + C::kFoldBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto relu_done = [&](int s) { return bar0 + 8u * (S + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * S + s); };
  auto accf = [&](int a) { return bar0 + 8u * (3 * S + a); };
  auto acce = [&](int a) { return bar0 + 8u * (3 * S + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (3 * S + 4);
  const uint32_t zfull = bar0 + 8u * (3 * S + 5);  // the ReLU warps wrote zpart
  const uint32_t zfree = bar0 + 8u * (3 * S + 6);  // warp 4 and the epilogue consumed zpart
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 7);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto a_buf = [&](int s) { return sbase + s * C::kStageBytes; };
  auto v_buf = [&](int s) { return sbase + s * C::kStageBytes + C::kABytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  TileCursor cur;
  cur.init(p.wp, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(relu_done(s), RW);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf(a), 1);
      mbar_init(acce(a), 4);
    }
    mbar_init(done_bar, 1);
    mbar_init(zfull, RW);
    mbar_init(zfree, 5);
    *abort = 0;
    fence_mbar_init();
  }
  if constexpr (C::kAAtoms > G::kAtoms) {
    // Rows d..127 of A: zero atoms that TMA never writes.
    const uint4 z = make_uint4(0, 0, 0, 0);
    constexpr int kPadBytes = (C::kAAtoms - G::kAtoms) * G::kAtomTileBytes;
    for (int s = 0; s < S; ++s)
      for (int o = threadIdx.x * 16; o < kPadBytes; o += C::kThreads * 16)
        st_shared_v4(a_buf(s) + G::kAtoms * G::kAtomTileBytes + o, z);
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
  // Launched as a programmatic dependent of whatever ran before it on the
  // stream: every global read or write below comes after that grid has
  // finished and its writes are visible (only the launch and this prologue
  // overlap its last CTAs).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      // gla_inject_stall (testing): CTA 0 withholds one tile, once
      long long stall = -1;
      if (blockIdx.x == 0 && g_gla_stall_tile >= 0) {
        stall = g_gla_stall_tile;
        g_gla_stall_tile = -1;
      }
      int64_t issued = 0;
      int b = 0, f = 0, h = 0;
      for (; cur.valid(); cur.advance(), ++issued) {
        const int s = static_cast<int>(issued % S);
        const uint32_t ph = static_cast<uint32_t>((issued / S) & 1);
        if (!mbar_wait(empty(s), ph ^ 1u, abort, kCode)) break;
        if (cur.first) unit_coords(cur.u, p.H, p.F, b, f, h);
        if (issued == stall) continue;  // nothing arrives on full(s) for this tile
        const int t = cur.t;
        mbar_arrive_expect_tx(full(s), 2u * G::kTileBytes);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a) {
          tma_load_5d(a_buf(s) + a * G::kAtomTileBytes, &tm_k, full(s), a * G::kAtomElems, h,
                      t * kTileTokens, f, b);
          tma_load_5d(v_buf(s) + a * G::kAtomTileBytes, &tm_v, full(s), a * G::kAtomElems, h,
                      t * kTileTokens, f, b);
        }
      }
      // Let every load still in flight land before the CTA can exit.
      for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
        mbar_wait_drain(full(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, true, true);
      int64_t i = 0, seg = 0;
      for (; cur.valid(); cur.advance(), ++i) {
        const bool first = cur.first;
        const bool last = cur.last;
        const int ab = static_cast<int>(seg & 1);
        if (first && !mbar_wait(acce(ab), static_cast<uint32_t>(((seg >> 1) & 1) ^ 1), abort, kCode))
          break;
        const int s = static_cast<int>(i % S);
        if (!mbar_wait(relu_done(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          const uint64_t ad = smem_desc(a_buf(s) + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          const uint64_t bd = smem_desc(v_buf(s) + kk * 2 * G::kGroupBytes, G::kAtomTileBytes,
                                        G::kGroupBytes, G::kLayout);
          mma_bf16(tmem + ab * AC, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
          if constexpr (kGram)  // M = phi(K)^T phi(K): B is the A tile itself (N = D)
            mma_bf16(tmem + ab * AC + D, ad, ad, idesc, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(empty(s));
        if (last) {
          mma_commit(accf(ab));
          ++seg;
        }
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- ReLU + normaliser sums
    constexpr int CPR = G::kChunksPerRow;     // 16-byte chunks per token row
    constexpr int RPP = RW * 32 / CPR;        // rows covered per pass of the ReLU warps
    constexpr int kPasses = kTileTokens / RPP;
    constexpr int CPA = G::kAtomElems / 8;    // chunks per swizzle row
    const int rt = threadIdx.x - 128;
    const int c = rt % CPR;
    const int r0 = rt / CPR;
    const uint32_t off0 = (c / CPA) * G::kAtomTileBytes + r0 * G::kRowBytes +
                          G::swz(r0, c % CPA) * 16;  // same swizzle slot for r0 + RPP*m
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = 0.f;
    int64_t i = 0;
    uint32_t zround = 0;
    RopeChunk rc{};
    RopeStep st{};
    int frame = 0;
    if constexpr (kRope) {
      rc = rope_chunk(p.rope, c);
      rope_step_init(p.rope, c, D / 2, st);
    }
    for (; cur.valid(); cur.advance(), ++i) {
      const int s = static_cast<int>(i % S);
      if (!warp_wait(full(s), static_cast<uint32_t>((i / S) & 1), abort, kCode)) break;
      const uint32_t base = a_buf(s) + off0;
      RopeRowPos rp{};
      if constexpr (kRope) {
        if (cur.first) frame = static_cast<int>((cur.u / p.H) % p.F);
        rp.start(cur.t * kTileTokens + r0, p.rope.grid_w);
        rope_coeffs(p.rope, rc, frame, rp, p.T, st.cs01, st.cs23);  // first row of the tile
      }
#pragma unroll
      for (int m = 0; m < kPasses; ++m) {
        const uint32_t addr = base + m * RPP * G::kRowBytes;
        uint4 w = ld_shared_v4(addr);
        relu8(w);
        if constexpr (kRope) {
          uint4 wr = w;
          rotate8(wr, st.cs01, st.cs23);
          st_shared_v4(addr, wr);
          rope_step_next(st, rp, p.rope.grid_w);
          rp.next(RPP, p.rope.grid_w);
        } else {
          st_shared_v4(addr, w);
        }
        z[0] += bf16lo_to_f32(w.x);
        z[1] += bf16hi_to_f32(w.x);
        z[2] += bf16lo_to_f32(w.y);
        z[3] += bf16hi_to_f32(w.y);
        z[4] += bf16lo_to_f32(w.z);
        z[5] += bf16hi_to_f32(w.z);
        z[6] += bf16lo_to_f32(w.w);
        z[7] += bf16hi_to_f32(w.w);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(relu_done(s));
      if (cur.last) {
        // Unit range ends: the column sums of phi(K) become row d of the
        // partial.  Each warp reduces its lanes, parks its sums in zpart[warp];
        // warp 4 adds the RW of them in a fixed order and writes the row.
#pragma unroll
        for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
          for (int e = 0; e < 8; ++e) z[e] += __shfl_xor_sync(0xffffffffu, z[e], o);
        if (zround > 0 && !warp_wait(zfree, (zround - 1) & 1u, abort, kCode)) break;
        if (lane < CPR) {
          float4* zp = reinterpret_cast<float4*>(zpart + (warp - 4) * D + lane * 8);
          zp[0] = make_float4(z[0], z[1], z[2], z[3]);
          zp[1] = make_float4(z[4], z[5], z[6], z[7]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(zfull);
        if (warp == 4) {
          if (!warp_wait(zfull, zround & 1u, abort, kCode)) break;
          if (!p.fold) {  // (a folding epilogue takes the sums itself)
            float* dst = p.partial + cur.slot() * static_cast<int64_t>(C::kPartialFloats) +
                         static_cast<int64_t>(D) * D;
            for (int col = lane; col < D; col += 32) {
              float zs = zpart[col];
#pragma unroll
              for (int w = 1; w < RW; ++w) zs += zpart[w * D + col];
              dst[col] = zs;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(zfree);
        }
        ++zround;
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = 0.f;
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // key feature i
    const bool has_row = q4 * 32 < D;
    int64_t seg = 0;
    for (; cur.valid(); cur.advance()) {
      if (!kRope && !kGram && p.fold && cur.first && cur.u < cur.U_full && has_row &&
          p.state_in != nullptr) {
        // a unit folded here: bring this warp's 32 state rows (16.5 KB) into
        // L2 while the unit's tiles stream, so that the fold reads them there
        int b, f, h;
        unit_coords(cur.u, p.H, p.F, b, f, h);
        const char* rows = reinterpret_cast<const char*>(
            p.state_in + (static_cast<int64_t>(b) * p.H + h) * D * (D + 1) +
            static_cast<int64_t>(q4 * 32) * (D + 1));
        for (int l = lane; l * 128 < 32 * (D + 1) * 4; l += 32)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rows + l * 128));
      }
      if (!cur.last) continue;
      const int ab = static_cast<int>(seg & 1);
      if (!warp_wait(accf(ab), static_cast<uint32_t>((seg >> 1) & 1), abort, kCode)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + ab * AC;
      float* dst = p.partial + cur.slot() * static_cast<int64_t>(C::kPartialFloats) + row;
      if (!kRope && !kGram && p.fold) {
        // ---- single frame: S = a S_in + dS for this CTA's units
        if (!warp_wait(zfull, static_cast<uint32_t>(seg & 1), abort, kCode)) break;
        float zs = 0.f;  // the normaliser column's entry of this key feature
        if (has_row) {
          zs = zpart[row];
#pragma unroll
          for (int w = 1; w < RW; ++w) zs += zpart[w * D + row];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(zfree);
        const int32_t u = cur.u;
        int b, f, h;
        unit_coords(u, p.H, p.F, b, f, h);
        const float a = 1.0f / (1.0f + expf(-__ldg(p.gate + u)));  // frame 0: gate index u
        // this warp's 32 key features i0 .. i0 + 31 of state (b, h), [d][d+1]
        const int64_t sbase = (static_cast<int64_t>(b) * p.H + h) * D * (D + 1) +
                              static_cast<int64_t>(q4 * 32) * (D + 1);
        uint8_t* img = p.image + static_cast<int64_t>(u) * G::kImageBytes +
                       (row / G::kAtomElems) * G::kImageAtomBytes + (row % 8) * 2;
        const int cin = (row % G::kAtomElems) / 8;
        float* tt = fold_t + q4 * 32 * 33;  // [32][33]: a 32 x 32 block, padded
        // one block of 32 value columns j0 ..: this thread holds dS[i0 + lane][j0 + c]
        // in dv[c]; S = a S_in + dS through the transpose tile so that state_in
        // and state_out move along their rows (lane = column) and the image
        // along its rows (lane = key feature)
        auto fold_block = [&](int j0, const float (&dv)[32]) {
#pragma unroll
          for (int c = 0; c < 32; ++c) tt[lane * 33 + c] = dv[c];
          __syncwarp();
          // the 32 state_in loads of the block in flight together
          float si[32];
#pragma unroll
          for (int r = 0; r < 32; ++r)
            si[r] = p.state_in != nullptr
                        ? p.state_in[sbase + static_cast<int64_t>(r) * (D + 1) + j0 + lane]
                        : 0.f;
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            const int64_t off = sbase + static_cast<int64_t>(r) * (D + 1) + j0 + lane;
            const float sv = fmaf(a, si[r], tt[r * 33 + lane]);
            if (p.state_out != nullptr) p.state_out[off] = sv;
            tt[r * 33 + lane] = sv;
          }
          __syncwarp();
#pragma unroll 8
          for (int c = 0; c < 32; ++c) {
            const int j = j0 + c;
            *reinterpret_cast<__nv_bfloat16*>(img + j * G::kRowBytes + G::swz(j, cin) * 16) =
                __float2bfloat16_rn(tt[lane * 33 + c]);
          }
          __syncwarp();
        };
        // the normaliser column j = d, one entry per thread
        auto fold_norm = [&](float dS) {
          const int64_t off = sbase + static_cast<int64_t>(lane) * (D + 1) + D;
          const float si = p.state_in != nullptr ? p.state_in[off] : 0.f;
          const float sv = fmaf(a, si, dS);
          if (p.state_out != nullptr) p.state_out[off] = sv;
          *reinterpret_cast<__nv_bfloat16*>(img + D * G::kRowBytes + G::swz(D, cin) * 16) =
              __float2bfloat16_rn(sv);
        };
        if (u < cur.U_full) {
          // the whole unit is this CTA's: fold from TMEM
          if (has_row) {
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t r[32];
              tmem_ld_32cols(tacc + cc * 32, r);
              tmem_wait_ld();
              float dv[32];
#pragma unroll
              for (int jj = 0; jj < 32; ++jj) dv[jj] = __uint_as_float(r[jj]);
              fold_block(cc * 32, dv);
            }
            fold_norm(zs);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acce(ab));
        } else {
          // a unit split over CTAs: this CTA's partial (the scan adds them up)
          if (has_row) {
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t r[32];
              tmem_ld_32cols(tacc + cc * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int jj = 0; jj < 32; ++jj) dst[(cc * 32 + jj) * D] = __uint_as_float(r[jj]);
            }
            dst[static_cast<int64_t>(D) * D] = zs;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acce(ab));
        }
        ++seg;
        continue;
      }
      if (has_row) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32cols(tacc + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) dst[(cc * 32 + jj) * D] = __uint_as_float(r[jj]);
        }
        if constexpr (kGram) {
          if (D == 128 && cur.u < cur.U_full) {
            // the whole unit: row i = row of M_f as the scan's A images
            uint8_t* img = reinterpret_cast<uint8_t*>(
                p.mpartial + cur.slot() * static_cast<int64_t>(D) * D);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t r[32];
              tmem_ld_32cols(tacc + D + cc * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(r[q * 8 + e]);
                uint4 hi, lo;
                split_bf16x8(x, hi, lo);
                const int off = GramImage<D>::offset(row, cc * 4 + q);
                *reinterpret_cast<uint4*>(img + off) = hi;
                *reinterpret_cast<uint4*>(img + GramImage<D>::kBytes + off) = lo;
              }
            }
          } else {
            float* mdst = p.mpartial + cur.slot() * static_cast<int64_t>(D) * D + row;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t r[32];
              tmem_ld_32cols(tacc + D + cc * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int jj = 0; jj < 32; ++jj) mdst[(cc * 32 + jj) * D] = __uint_as_float(r[jj]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(acce(ab));
        mbar_arrive(zfree);  // (the normaliser sums are warp 4's here)
      }
      ++seg;
    }
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
