// gla_softmax_anchor.cuh -- the softmax anchor layer (attention sinks + a
// local window of frames) on tcgen05.
//
// The SANA-Video 2.0 pages put a gated-softmax anchor after every three
// linear layers; the SANA-WM pages give the softmax layers attention-sink
// tokens and a local temporal window so that memory and per-chunk latency stay
// constant over long rollouts.  This library's reading, per (b, h): the
// queries of frame f attend to all tokens of frames max(0, f-W+1) .. f and to
// the first n_sink tokens of the sequence that precede that window, with
// scores q . k / sqrt(d); out = sigmoid(z) * softmax-weighted sum of v (z an
// optional per-element gate).
//
// One work unit = 128 query tokens of one (b, f, h).  Its key tiles (128 keys
// of one frame, the frame's last tile ragged) are walked once, online:
//   S = Q K^T into TMEM (two buffers); the softmax warps write
//   P = 2^((S - m) log2(e) / sqrt(d)) in bf16 back into the S buffer they
//   just read (two bf16 per 32-bit column, each key half into the first half
//   of its own columns) and sum l = sum P; O += P V accumulates in TMEM with
//   P as the MMA's A operand straight from TMEM.
// The reference maximum m of a row moves lazily: only when a tile's maximum
// exceeds it by more than 2^kRescaleLog2 in P, and then the row of O and l are
// scaled by the ratio (after the previous P V has completed); otherwise P is
// at most 2^kRescaleLog2 and the reference stays.  With scores of unit scale
// this happens on a handful of tiles per unit.
// Softmax warp w owns the query rows 32 (w % 4) .. + 31 (its TMEM lane
// quarter) and the keys 64 (w / 4) .. + 63 of every tile; each key half keeps
// its own m, l and O accumulator (P V is issued as two K = 64 halves), so the
// two warps of a row quarter never wait on each other per tile.  They swap
// (m, l) once per unit, through their own columns of the unit's last S buffer,
// and the epilogue combines out = sigmoid(z) (O_0 f_0 + O_1 f_1) / (l_0 f_0 +
// l_1 f_1), f_c = 2^(m_c - max(m_0, m_1)) in the scaled units.
// The softmax is bound by instruction issue and the MUFU exponential unit:
// it scales and shifts the scores and sums P on packed fp32 pairs
// (fma / add .f32x2), takes the tile maximum with a three-input max, and
// computes one pair of exponentials in four on the FMA pipe (exp2_poly3_x2),
// the rest with ex2.approx.
// The MMA issuers run one tile ahead: S of tile j+1 is issued before P V of
// tile j, so the tensor core computes the next scores while the softmax warps
// exponentiate.  Ring order of the key/value tiles: K0 K1 V0 K2 V1 ..
// K(n-1) V(n-2) V(n-1), the order in which they are consumed.
//   S:  A = Q [M = 128 queries, K = d] K-major,   B = K tile [N = 128 keys] K-major
//   PV: A = P [M = 128 queries, K = 64 keys] in TMEM, B = V rows [N = d] MN-major
// Warp roles: 0-7 softmax / epilogue, 8 TMA, 9 and 10 MMA.  A tcgen05.mma
// issue returns only about when the tensor core takes the instruction, so a
// lone issuing thread leaves the tensor core idle while it waits on barriers
// and commits; two issuers overlap that bookkeeping with each other's MMAs:
// issuer 0 takes every S = Q K^T, issuer 1 every O += P V (one thread, so the
// accumulation into O keeps its order).
#pragma once

#include "gla_common.cuh"
#include "gla_increment.cuh"  // warp_wait, unit_coords
#include "sm100_ptx.cuh"

namespace gla {

struct AnchorParams {
  int H, F, T;       // heads, frames, tokens per frame
  int window;        // W >= 1 frames
  int n_sink;        // sink tokens at the start of the sequence
  int units;         // B * F * H * tiles per frame
  float scale_log2;  // log2(e) / sqrt(d)
  int has_gate;
  // Rollout step (step != 0): q, k, v, z and out hold one frame (F == 1), the
  // frame `frame` of the sequence; the earlier frames of its window come from
  // a window cache (win_frames frames, oldest first) and the sink tokens
  // from a sink cache (the first n_sink tokens of the sequence).  The key
  // tiles are the same, in the same order, as for that frame in a call over
  // the whole sequence.
  int step;
  int frame;
};

// The key tiles of the queries of frame f, in order: the sink tokens that
// precede the window (frames 0 .., the last one possibly partial), then the
// window's frames.  Each tile is (frame, first token t0, valid rows).
struct KeyTiles {
  int T, f, w_lo_frame, s_hi;  // s_hi: sink tokens [0, s_hi), s_hi <= w_lo_frame * T
  int fr, t0, valid, end_t;    // current tile
  bool in_sink, done;

  __device__ void init(int T_, int f_, int window, int n_sink) {
    T = T_;
    f = f_;
    w_lo_frame = f - window + 1 > 0 ? f - window + 1 : 0;
    const int w_lo = w_lo_frame * T;
    s_hi = n_sink < w_lo ? n_sink : w_lo;
    done = false;
    if (s_hi > 0) {
      in_sink = true;
      fr = 0;
    } else {
      in_sink = false;
      fr = w_lo_frame;
    }
    t0 = 0;
    set_end();
    if (end_t <= 0) done = true;  // T == 0
    valid = end_t - t0 < kTileTokens ? end_t - t0 : kTileTokens;
  }
  __device__ void set_end() {
    end_t = in_sink ? ((s_hi - fr * T) < T ? s_hi - fr * T : T) : T;
  }
  __device__ void advance() {
    t0 += kTileTokens;
    if (t0 >= end_t) {
      t0 = 0;
      ++fr;
      if (in_sink && fr * T >= s_hi) {
        in_sink = false;
        fr = w_lo_frame;
      }
      if (!in_sink && fr > f) {
        done = true;
        return;
      }
      set_end();
    }
    valid = end_t - t0 < kTileTokens ? end_t - t0 : kTileTokens;
  }
};

// 2^x on the FMA pipe, for part of the exponentials of P (the MUFU unit that
// runs ex2.approx does 16 per clock per SM and bounds the softmax otherwise).
// Range reduction: adding 1.5 * 2^23 rounds x to the nearest integer n in the
// low mantissa bits, r = x - n lies in [-1/2, 1/2]; 2^r by a degree-3
// polynomial fitted to 2^r on that interval (iteratively reweighted least
// squares towards the minimax relative error: 7.5e-5, far below the bf16
// rounding of P); n is added to the exponent field.  x is clamped at -126, so
// masked keys (x = -inf) give about 1e-38 instead of 0, which no sum notices.
constexpr float kExp2C0 = 0.9999281167984009f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.24261054396629333f;
constexpr float kExp2C3 = 0.05517132207751274f;

__device__ __forceinline__ float exp2_poly3(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23
  const float r = x - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(kExp2C3, r, kExp2C2), r, kExp2C1), r, kExp2C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same for two lanes with the packed pair arithmetic.
__device__ __forceinline__ void exp2_poly3_x2(float a0, float a1, float& x0, float& x1) {
  const uint64_t x = f2_pack(fmaxf(a0, -126.0f), fmaxf(a1, -126.0f));
  const uint64_t t = f2_add(x, f2_pack(12582912.0f, 12582912.0f));
  const uint64_t r = f2_sub(x, f2_sub(t, f2_pack(12582912.0f, 12582912.0f)));
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), r, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, r, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, r, f2_pack(kExp2C0, kExp2C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  x0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  x1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

template <int D>
struct AnchorCfg {
  using G = Geo<D>;
  static_assert(D == 128, "the softmax anchor kernel is built for d = 128");
  static constexpr int kStages = 5;                 // K / V tile ring
  static constexpr int kTileBytes = G::kTileBytes;  // 32 KB
  static constexpr int kThreads = 352;
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kTmemCols = 512;             // S x 2 (256) + O of each key half (256)
  static constexpr int kAccO = 256;                 // O of key half c at kAccO + 128 c
  static constexpr float kRescaleLog2 = 8.0f;       // P <= 2^8 between rescales
  static constexpr int kPolyPairs = 1;              // of each 4 pairs of exponentials, on the
                                                    // FMA pipe
  static constexpr int kBarCount = 2 * kStages + 16;
  // Q, gate / output, ring
  static constexpr int kSmemBytes = 1024 + (2 + kStages) * kTileBytes + kBarCount * 8 + 16;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// Key / value sources of a rollout step (unused by a whole-sequence call):
// the sink cache [B, n_sink, H, d] and the window cache [B, frames * T, H, d].
struct AnchorCaches {
  CUtensorMap ks, vs, kw, vw;
};

template <int D>
__global__ void __launch_bounds__(352, 1)
    gla_softmax_anchor_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ CUtensorMap tm_z,
                              const __grid_constant__ CUtensorMap tm_out,
                              const __grid_constant__ AnchorCaches caches, const AnchorParams p) {
  using G = Geo<D>;
  using C = AnchorCfg<D>;
  constexpr int S = C::kStages;
  constexpr unsigned kCode = 128u;
  constexpr int KPA = G::kAtomElems / 16;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_buf = sbase;
  const uint32_t o_buf = sbase + C::kTileBytes;  // gate in, output out
  auto ring = [&](int s) { return sbase + (2 + s) * C::kTileBytes; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (2 + S) * C::kTileBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto rfull = [&](int s) { return bar0 + 8u * s; };
  auto rempty = [&](int s) { return bar0 + 8u * (S + s); };
  const uint32_t qfull = bar0 + 8u * (2 * S + 0);
  const uint32_t qempty = bar0 + 8u * (2 * S + 1);
  // per S buffer b: S landed (sfull), the softmax warps are done with its
  // scores and, on a unit's last tile, with the (m, l) exchange (sfree), P is
  // written over it (pfull), the P V that read that P is done (pfree)
  auto sfull = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
  auto sfree = [&](int b) { return bar0 + 8u * (2 * S + 4 + b); };
  auto pfull = [&](int b) { return bar0 + 8u * (2 * S + 6 + b); };
  auto pfree = [&](int b) { return bar0 + 8u * (2 * S + 8 + b); };
  const uint32_t ofull = bar0 + 8u * (2 * S + 10);
  const uint32_t ofree = bar0 + 8u * (2 * S + 11);
  const uint32_t zfull = bar0 + 8u * (2 * S + 12);
  const uint32_t zfree = bar0 + 8u * (2 * S + 13);
  const uint32_t done_bar = bar0 + 8u * (2 * S + 14);
  const uint32_t xbar = bar0 + 8u * (2 * S + 15);  // (m, l) exchange of the two key halves
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBarCount);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tpf = (p.T + kTileTokens - 1) / kTileTokens;  // query tiles per frame

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(rfull(s), 1);
      mbar_init(rempty(s), 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sfree(b), C::kSoftmaxWarps);
      mbar_init(pfull(b), C::kSoftmaxWarps);
      mbar_init(pfree(b), 1);
    }
    mbar_init(ofull, 1);
    mbar_init(ofree, C::kSoftmaxWarps);
    mbar_init(zfull, 1);
    mbar_init(zfree, C::kSoftmaxWarps);
    mbar_init(done_bar, 2);
    mbar_init(xbar, C::kSoftmaxWarps);
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

  // unit -> (b, f, h, query tile): unit = ((b * F + f) * H + h) * tpf + qt
  auto coords = [&](int unit, int& b, int& f, int& h, int& qt) {
    qt = unit % tpf;
    const int u = unit / tpf;
    unit_coords(u, p.H, p.F, b, f, h);
  };

  if (warp == C::kSoftmaxWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int64_t n = 0;  // ring tiles issued
      int64_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++it) {
        int b, f, h, qt;
        coords(unit, b, f, h, qt);
        const uint32_t ph = static_cast<uint32_t>(it & 1);
        if (!mbar_wait(qempty, ph ^ 1u, abort, kCode)) break;
        mbar_arrive_expect_tx(qfull, G::kTileBytes);
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_5d(q_buf + a * G::kAtomTileBytes, &tm_q, qfull, a * G::kAtomElems, h,
                      qt * kTileTokens, f, b);
        if (p.has_gate) {
          if (!mbar_wait(zfree, ph ^ 1u, abort, kCode)) break;
          mbar_arrive_expect_tx(zfull, G::kTileBytes);
          for (int a = 0; a < G::kAtoms; ++a)
            tma_load_5d(o_buf + a * G::kAtomTileBytes, &tm_z, zfull, a * G::kAtomElems, h,
                        qt * kTileTokens, f, b);
        }
        // one ring tile: K or V rows [t0, t0 + 128) of frame fr (of the
        // sequence; a rollout step reads the caches for earlier frames)
        auto load = [&](bool is_v, const KeyTiles& t) {
          const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
          int fr = t.fr, t0 = t.t0;
          if (p.step) {
            if (t.in_sink) {  // sink tokens fr * T + t0 .. of the sink cache
              tm = is_v ? &caches.vs : &caches.ks;
              t0 += fr * p.T;
              fr = 0;
            } else if (t.fr < t.f) {  // an earlier frame of the window
              tm = is_v ? &caches.vw : &caches.kw;
              fr = t.fr - t.w_lo_frame;
            } else {
              fr = 0;
            }
          }
          const int s = static_cast<int>(n % S);
          if (!mbar_wait(rempty(s), static_cast<uint32_t>(((n / S) & 1) ^ 1), abort, kCode))
            return false;
          mbar_arrive_expect_tx(rfull(s), G::kTileBytes);
          for (int a = 0; a < G::kAtoms; ++a)
            tma_load_5d(ring(s) + a * G::kAtomTileBytes, tm, rfull(s), a * G::kAtomElems, h, t0,
                        fr, b);
          ++n;
          return true;
        };
        KeyTiles kt, prev;
        bool has_prev = false;  // the previous tile, whose V follows this tile's K
        for (kt.init(p.T, p.step ? p.frame : f, p.window, p.n_sink); ok && !kt.done;
             kt.advance()) {
          ok = load(false, kt);
          if (ok && has_prev) ok = load(true, prev);
          prev = kt;
          has_prev = true;
        }
        if (ok && has_prev) ok = load(true, prev);
      }
      for (int64_t i = (n > S ? n - S : 0); i < n; ++i)
        mbar_wait_drain(rfull(static_cast<int>(i % S)), static_cast<uint32_t>((i / S) & 1));
    }
  } else if (warp == C::kSoftmaxWarps + 1 || warp == C::kSoftmaxWarps + 2) {
    // ------------------------------------------------------------ MMA issuers
    const uint32_t me = static_cast<uint32_t>(warp - C::kSoftmaxWarps - 1);
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTileTokens, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      // Operand descriptors are built once; a K step or another buffer only
      // moves the start address field (address >> 4, low 14 bits), so the
      // issue loop adds compile-time offsets (shared memory is < 256 KB, no
      // carry leaves the field).
      constexpr uint64_t kBufStep = C::kTileBytes >> 4;
      const uint64_t qd = smem_desc(q_buf, 16, G::kGroupBytes, G::kLayout);
      const uint64_t kd = smem_desc(ring(0), 16, G::kGroupBytes, G::kLayout);
      const uint64_t vd = smem_desc(ring(0), G::kAtomTileBytes, G::kGroupBytes, G::kLayout);
      uint32_t rs = 0, rph = 0;  // ring slot and phase of the next tile consumed
      uint32_t ns = 0, np = 0;   // S tiles, P tiles
      auto ring_next = [&]() {
        if (++rs == static_cast<uint32_t>(S)) {
          rs = 0;
          rph ^= 1u;
        }
      };
      int64_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++it) {
        int b, f, h, qt;
        coords(unit, b, f, h, qt);
        const uint32_t ph = static_cast<uint32_t>(it & 1);
        if (!mbar_wait(qfull, ph, abort, kCode)) break;
        // issuer 0: S = Q K^T of the next ring tile into S buffer ns % 2
        // (the buffer also held P of tile ns - 2: wait for that P V too)
        auto issue_s = [&]() {
          const uint32_t sb = ns & 1u;
          if (!mbar_wait(sfree(sb), ((ns >> 1) & 1u) ^ 1u, abort, kCode) ||
              !mbar_wait(pfree(sb), ((ns >> 1) & 1u) ^ 1u, abort, kCode) ||
              !mbar_wait(rfull(rs), rph, abort, kCode))
            return false;
          tc_fence_after();
          const uint64_t bd0 = kd + rs * kBufStep;
          const uint32_t dt = tmem + sb * kTileTokens;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off =
                static_cast<uint64_t>(((kk / KPA) * G::kAtomTileBytes + (kk % KPA) * 32) >> 4);
            mma_bf16(dt, qd + off, bd0 + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(sfull(sb));
          mma_commit(rempty(rs));
          ring_next();
          ++ns;
          return true;
        };
        // issuer 1: O_c += P[:, 64 c ..] V[64 c .., :] for both key halves c, P
        // in S buffer np % 2 (key half c at its columns 64 c .. + 31) and V the
        // next ring tile
        auto issue_pv = [&](bool first) {
          const uint32_t pb = np & 1u;
          if (!mbar_wait(pfull(pb), (np >> 1) & 1u, abort, kCode) ||
              !mbar_wait(rfull(rs), rph, abort, kCode))
            return false;
          if (first && !mbar_wait(ofree, ph ^ 1u, abort, kCode)) return false;
          tc_fence_after();
          const uint32_t pa = tmem + pb * kTileTokens;
          const uint64_t bd0 = vd + rs * kBufStep;
#pragma unroll
          for (int kk = 0; kk < kTileTokens / 16; ++kk) {
            const uint32_t acol = (kk / KPA) * 64 + (kk % KPA) * 8;  // 16 keys = 8 columns
            const uint64_t boff = static_cast<uint64_t>((kk * 2 * G::kGroupBytes) >> 4);
            mma_bf16_ts(tmem + C::kAccO + (kk / KPA) * D, pa + acol, bd0 + boff, idesc_o,
                        (first && kk % KPA == 0) ? 0u : 1u);
          }
          mma_commit(pfree(pb));
          mma_commit(rempty(rs));
          ring_next();
          ++np;
          return true;
        };
        // a tile the other issuer takes: only the counters move
        auto skip_s = [&]() {
          ring_next();
          ++ns;
          return true;
        };
        auto skip_pv = [&]() {
          ring_next();
          ++np;
          return true;
        };
        KeyTiles kt;
        kt.init(p.T, p.step ? p.frame : f, p.window, p.n_sink);
        if (!kt.done) {
          ok = me == 0 ? issue_s() : skip_s();
          for (bool first = true; ok; first = false) {
            kt.advance();
            const bool more = !kt.done;
            if (more) ok = me == 0 ? issue_s() : skip_s();
            if (ok) ok = me == 1 ? issue_pv(first) : skip_pv();
            if (!more) break;
          }
        }
        if (!ok) break;
        mma_commit(qempty);              // this issuer's reads of Q are done
        if (me == 1) mma_commit(ofull);  // O of this unit complete
      }
      mma_commit(done_bar);
      mbar_wait_drain(done_bar, 0);
    }
  } else {
    // -------------------------------------------------- softmax and epilogue
    const int q4 = warp & 3;          // TMEM lane quarter: query rows 32 q4 ..
    const int hc = warp >> 2;         // key half of the tiles, output columns 64 hc ..
    const int row = q4 * 32 + lane;   // query within the tile
    const int c0 = hc * 64;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const float sl2 = p.scale_log2;
    int64_t ns = 0, np = 0, it = 0;
    for (int unit = blockIdx.x; unit < p.units; unit += gridDim.x, ++it) {
      int b, f, h, qt;
      coords(unit, b, f, h, qt);
      const uint32_t ph = static_cast<uint32_t>(it & 1);
      float m = -INFINITY, l = 0.f;  // this key half's reference maximum and sum
      float mo = -INFINITY, lo = 0.f;  // the other half's, after the exchange
      bool ok = true;
      KeyTiles kt;
      kt.init(p.T, p.step ? p.frame : f, p.window, p.n_sink);
      for (bool first = true; !kt.done; first = false) {
        const int sb = static_cast<int>(ns & 1);
        KeyTiles nx = kt;
        nx.advance();
        const bool last = nx.done;
        if (!warp_wait_fast(sfull(sb), static_cast<uint32_t>((ns >> 1) & 1), abort, kCode)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ra[32], rb[32];  // keys c0 .. c0 + 31, c0 + 32 .. c0 + 63
        const uint32_t ts = tmem + lane_base + sb * kTileTokens + c0;
        tmem_ld_32cols(ts, ra);
        tmem_ld_32cols(ts + 32, rb);
        tmem_wait_ld();
        if (kt.valid < c0 + 64) {  // keys past the tile's end: S = -inf
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (c0 + e >= kt.valid) ra[e] = __float_as_uint(-INFINITY);
            if (c0 + 32 + e >= kt.valid) rb[e] = __float_as_uint(-INFINITY);
          }
        }
        if (!last) {  // the unit's last S buffer carries the (m, l) exchange
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sfree(sb));
        }
        float mt;
        {
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mx[e & 3] = fmax3(mx[e & 3], __uint_as_float(ra[e]), __uint_as_float(rb[e]));
          mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        }
        bool grow = false;
        if (first || m == -INFINITY)
          m = mt;  // no P of this row's half has been non-zero yet: O and l are zero
        else
          grow = (mt - m) * sl2 > C::kRescaleLog2;
        if (!first) {  // warp-uniform
          if (__any_sync(0xffffffffu, grow)) {
            // scale this warp's rows of O_hc once the previous P V is done
            const uint32_t pp = static_cast<uint32_t>(np - 1);
            if (!warp_wait(pfree(static_cast<int>(pp & 1u)), (pp >> 1) & 1u, abort, kCode)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float fct = grow ? ex2_approx((m - mt) * sl2) : 1.0f;
            if (grow) {
              l *= fct;
              m = mt;
            }
            const uint32_t to = tmem + lane_base + C::kAccO + hc * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld_32cols(to + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * fct);
              tmem_st_32cols(to + cc * 32, o);
            }
            tmem_wait_st();
          }
        }
        // P = 2^((S - m) scale log2 e) in bf16 (masked keys give 0), written
        // over this half's S columns (S of this buffer landed after the P V
        // that last read it, so the columns are free)
        const int pb = static_cast<int>(np & 1);
        const float ms = m == -INFINITY ? 0.f : m * sl2;
        uint32_t pw[32];
        const uint64_t sc2 = f2_pack(sl2, sl2), sh2 = f2_pack(-ms, -ms);
        uint64_t ls2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};  // pair-wise row sums
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int e = ch * 8 + 2 * e2;
            const float s0 = __uint_as_float(e < 32 ? ra[e] : rb[e - 32]);
            const float s1 = __uint_as_float(e < 32 ? ra[e + 1] : rb[e - 31]);
            float a0, a1, x0, x1;
            f2_unpack(f2_fma(f2_pack(s0, s1), sc2, sh2), a0, a1);
            if (e2 < C::kPolyPairs) {
              exp2_poly3_x2(a0, a1, x0, x1);
            } else {
              x0 = ex2_approx(a0);
              x1 = ex2_approx(a1);
            }
            ls2[e2 & 1] = f2_add(ls2[e2 & 1], f2_pack(x0, x1));
            pw[ch * 4 + e2] = pack_bf16x2(x0, x1);
          }
        }
        tmem_st_32cols(tmem + lane_base + sb * kTileTokens + c0, pw);
        tmem_wait_st();
        {
          float l0, l1, l2, l3;
          f2_unpack(ls2[0], l0, l1);
          f2_unpack(ls2[1], l2, l3);
          l += (l0 + l1) + (l2 + l3);
        }
        tc_fence_before();  // orders P's (and a rescale's) TMEM stores before the P V
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull(pb));
        ++np;
        if (last) {
          // swap (m, l) with the other key half through this half's own
          // columns of the S buffer just read (past its P), then release it
          const uint32_t mine = tmem + lane_base + sb * kTileTokens + c0 + 32;
          const uint32_t other = tmem + lane_base + sb * kTileTokens + (c0 ^ 64) + 32;
          tmem_st_1col(mine, __float_as_uint(m));
          tmem_st_1col(mine + 1, __float_as_uint(l));
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(xbar);
          if (!warp_wait(xbar, ph, abort, kCode)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t v0, v1;
          tmem_ld_1col(other, v0);
          tmem_ld_1col(other + 1, v1);
          tmem_wait_ld();
          mo = __uint_as_float(v0);
          lo = __uint_as_float(v1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sfree(sb));
        }
        ++ns;
        kt = nx;
      }
      if (!ok) break;
      // ---- epilogue: out = sigmoid(z) (O_0 f_0 + O_1 f_1) / (l_0 f_0 + l_1 f_1)
      const float mm = fmaxf(m, mo);
      const float f_me = m == -INFINITY ? 0.f : ex2_approx((m - mm) * sl2);
      const float f_ot = mo == -INFINITY ? 0.f : ex2_approx((mo - mm) * sl2);
      const float f0 = hc == 0 ? f_me : f_ot, f1 = hc == 0 ? f_ot : f_me;
      const float rl = 1.0f / (l * f_me + lo * f_ot);
      if (!warp_wait(ofull, ph, abort, kCode)) break;
      if (p.has_gate && !warp_wait(zfull, ph, abort, kCode)) break;
      tc_fence_after();
      if (lane == 0) bulk_wait_group_read<0>();  // the previous output left o_buf
      __syncwarp();
      const uint32_t obase = o_buf + hc * G::kAtomTileBytes + row * G::kRowBytes;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t ra[32], rb[32];  // O_0 and O_1, output columns c0 + 32 cc ..
        const uint32_t to = tmem + lane_base + C::kAccO + c0 + cc * 32;
        tmem_ld_32cols(to, ra);
        tmem_ld_32cols(to + D, rb);
        tmem_wait_ld();
        if (cc == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(ofree);  // O read into registers
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint32_t addr = obase + G::swz(row, cc * 4 + ch) * 16;
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            x[e] = (__uint_as_float(ra[ch * 8 + e]) * f0 + __uint_as_float(rb[ch * 8 + e]) * f1) *
                   rl;
          if (p.has_gate) {
            const uint4 zw = ld_shared_v4(addr);
            const uint32_t zz[4] = {zw.x, zw.y, zw.z, zw.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float z = (e & 1) ? bf16hi_to_f32(zz[e >> 1]) : bf16lo_to_f32(zz[e >> 1]);
              x[e] *= 1.0f / (1.0f + expf(-z));
            }
          }
          uint4 w;
          w.x = pack_bf16x2(x[0], x[1]);
          w.y = pack_bf16x2(x[2], x[3]);
          w.z = pack_bf16x2(x[4], x[5]);
          w.w = pack_bf16x2(x[6], x[7]);
          st_shared_v4(addr, w);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int tok0 = qt * kTileTokens + q4 * 32;
        if (tok0 < p.T)
          tma_store_5d(&tm_out, o_buf + hc * G::kAtomTileBytes + q4 * 32 * G::kRowBytes,
                       hc * G::kAtomElems, h, tok0, f, b);
        bulk_commit_group();
        bulk_wait_group_read<0>();  // the next unit's gate may land in o_buf
        if (p.has_gate) mbar_arrive(zfree);
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
