// gla_api.cu -- C ABI of the gated linear attention library (see gla.h).
//
// gla_forward validates its arguments (no CUDA call before that), takes a
// stream-ordered workspace, builds the TMA tensor maps of q, k, v and out,
// and enqueues the three kernels on the caller's stream:
//   1. gla_increment_kernel  dS_f partials  (tcgen05, TMA, ReLU fused)
//   2. gla_scan_kernel       S_f = a_f S_{f-1} + dS_f, state_out, bf16 S_f^T images
//   3. gla_output_kernel     out = phi(q) S_f / (phi(q) S_f[:, d] + eps)   (tcgen05)
// gla_backward (d = 128) recomputes the forward states and enqueues
//   1. gla_increment_kernel  dS_f partials
//   2. gla_scan_kernel       S_f (fp32, kept) and bf16 S_f^T images
//   3. gla_bwd_q_kernel      dq and the local state gradients L_f   (tcgen05)
//   4. gla_scan_bwd_kernel   G_f = L_f + a_{f+1} G_{f+1}, dstate_in, da_f partial sums,
//                            bf16 G_f^T images
//   5. gla_dgate_kernel      dg = a (1 - a) da
//   6. gla_bwd_kv_kernel     dk, dv                                   (tcgen05)
// gla_forward_gdn (the frame-wise delta-rule variant) enqueues
//   1. gla_increment_kernel  dS_f partials and M_f = phi(K_f)^T phi(K_f)    (tcgen05;
//                            at d = 128 a whole unit's M_f as bf16 hi/lo MMA operand images)
//   1b. for units split over several CTAs: gla_gdn_tail_reduce_kernel (d = 128) or
//       gla_gram_reduce_kernel (d = 32, 64)
//   2. gla_gdn_scan_tc_kernel (d = 128, the product M_f S_{f-1} on tcgen05) or
//      gla_gdn_scan_kernel (d = 32, 64): S_f = a_f (S_{f-1} - beta_f M_f S_{f-1}) + beta_f dS_f
//   3. gla_output_kernel     as gla_forward
// gla_softmax_anchor (d = 128) runs gla_softmax_anchor_kernel: one online pass
// over the key tiles of sinks + window, S = Q K^T and O += P V on tcgen05
// with the running maxima and sums in the softmax warps.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gla.h"
#include "gla_bwd_kv.cuh"
#include "gla_bwd_q.cuh"
#include "gla_common.cuh"
#include "gla_gdn_scan.cuh"
#include "gla_increment.cuh"
#include "gla_output.cuh"
#include "gla_rope.cuh"
#include "gla_scan.cuh"
#include "gla_scan_bwd.cuh"
#include "gla_softmax_anchor.cuh"
#include "sm100_ptx.cuh"

namespace {

// Partial slices in flight per scan block over a sequence of frames (three
// blocks of 74 KB share an SM at 4).
constexpr int kScanStages = 4;


using gla::Geo;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int major = 0;
  void* scratch = nullptr;  // device address of g_gla_scratch (gla_forward_noalloc)
};

// Fixed scratch of gla_forward_noalloc: a file-scope device array that every
// device which loads this library holds until the process exits.  In host
// code its name is only a stand-in; the kernels get the device address that
// cudaGetSymbolAddress returns for the current device.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_gla_scratch[kNoAllocScratchBytes];

struct FixedScratch {
  uint8_t* ptr;
  size_t bytes;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
// Per-device stream-ordered pool for gla_forward's workspace.  Its release
// threshold is unbounded, so memory freed at the end of a call stays mapped
// for the next call instead of going back to the driver at the caller's next
// synchronisation (re-mapping hundreds of MB costs tens of milliseconds).
// gla_trim_workspace() returns it.
cudaMemPool_t g_pool[kMaxDevices] = {};

cudaMemPool_t workspace_pool() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_pool[dev] == nullptr) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    uint64_t keep = ~uint64_t(0);
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = pool;
  }
  return g_pool[dev];
}
// gla_inject_alloc_failure (testing): workspace allocations still to fail.
int g_fail_allocs = 0;

// Stream-ordered workspace of `bytes` from the device's pool; GLA_ERR_ALLOC
// (nothing enqueued) when the pool cannot provide it.
int take_workspace(int64_t bytes, cudaStream_t stream, uint8_t** ws) {
  *ws = nullptr;
  if (bytes <= 0) return GLA_OK;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_fail_allocs > 0) {
      --g_fail_allocs;
      return GLA_ERR_ALLOC;
    }
  }
  cudaMemPool_t pool = workspace_pool();
  if (pool == nullptr || cudaMallocFromPoolAsync(reinterpret_cast<void**>(ws),
                                                 static_cast<size_t>(bytes), pool,
                                                 stream) != cudaSuccess) {
    cudaGetLastError();
    *ws = nullptr;
    return GLA_ERR_ALLOC;
  }
  return GLA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

template <int D>
cudaError_t set_smem_attrs() {
  cudaError_t e = cudaFuncSetAttribute(gla::gla_increment_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       gla::IncCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_output_kernel<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::OutCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_scan_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::ScanCfg<D, 1>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_scan_kernel<D, kScanStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::ScanCfg<D, kScanStages>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_increment_kernel<D, false, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::IncCfg<D, false, true>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_gdn_scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::GdnScanCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  if constexpr (D == 128) {
    e = cudaFuncSetAttribute(gla::gla_softmax_anchor_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gla::AnchorCfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gla::gla_gdn_scan_tc_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gla::GdnTcCfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(gla::gla_increment_kernel<D, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::IncCfg<D, true>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_output_kernel<D, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::OutCfg<D, true>::kSmemBytes);
  if (e != cudaSuccess || D != 128) return e;
  e = cudaFuncSetAttribute(gla::gla_bwd_q_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::BwdQCfg<128>::kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla::gla_bwd_kv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           gla::BwdKVCfg<128>::kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(gla::gla_scan_bwd_kernel<128>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              gla::ScanBwdCfg<128>::kSmemBytes);
}

// Per-device one-time set-up: SM count, architecture check, kernel attributes,
// the driver's tensor-map encoder.
int device_setup(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return GLA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return GLA_ERR_DEVICE;
    if (prop.major != 10) return GLA_ERR_DEVICE;
    if (set_smem_attrs<32>() != cudaSuccess || set_smem_attrs<64>() != cudaSuccess ||
        set_smem_attrs<128>() != cudaSuccess)
      return GLA_ERR_LAUNCH;
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return GLA_ERR_DEVICE;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    di.sms = prop.multiProcessorCount;
    di.major = prop.major;
    di.ready = true;
  }
  *out = di;
  return GLA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 5-D view (d, H, T, F, B) of a bf16 [B, F*T, H, d] tensor; box = one swizzle
// atom of features x `box_rows` tokens of one head of one frame.
// Tensor map of a bf16 [B, F*T, H, d] tensor with boxes of `box_rows` tokens
// x `box_cols` features (0: one swizzle atom, 64 features at d >= 64, else
// 32); 32-feature boxes use the 64-byte swizzle, 64-feature boxes 128-byte.
int encode_map(CUtensorMap* m, const void* base, int d, int H, int T, int F, int B, int box_rows,
               int box_cols = 0) {
  const int atom = box_cols > 0 ? box_cols : (d >= 64 ? 64 : 32);
  const cuuint64_t e = 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(F),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[4] = {d * e, static_cast<cuuint64_t>(H) * d * e,
                           static_cast<cuuint64_t>(T) * H * d * e,
                           static_cast<cuuint64_t>(F) * T * H * d * e};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(atom), 1, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        atom == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GLA_OK : GLA_ERR_LAUNCH;
}

struct Args {
  const void *q, *k, *v;
  const float* g;
  const float* s_in;
  float* s_out;
  void* out;
  int B, H, F, T, d;
  float eps;
  cudaStream_t stream;
  const gla_rope_config* rope = nullptr;  // rotary variant when set
  const float* beta = nullptr;            // delta-rule variant: [B, F, H] write-strength logits
  uint8_t* saved = nullptr;               // training forward: the context for the backward
};


// Host-only checks of a rotary configuration; no CUDA call.
int validate_rope(const gla_rope_config* r, int d) {
  if (r == nullptr) return GLA_ERR_NULL;
  const int dims[3] = {r->dim_t, r->dim_y, r->dim_x};
  for (int n : dims)
    if (n < 0 || n % 8 != 0) return GLA_ERR_ROPE;
  if (dims[0] + dims[1] + dims[2] != d) return GLA_ERR_ROPE;
  if (r->grid_w < 1 || r->frame_offset < 0 || r->frame_offset > (1 << 24)) return GLA_ERR_ROPE;
  if (!(r->theta > 0.0f) || r->theta > 3.0e38f) return GLA_ERR_ROPE;  // rejects NaN and inf
  return GLA_OK;
}

// Host-only checks; no CUDA call.
int validate(const Args& a) {
  if (a.d != 32 && a.d != 64 && a.d != 128) return GLA_ERR_UNSUPPORTED_D;
  if (a.B < 0 || a.H < 0 || a.F < 0 || a.T < 0) return GLA_ERR_SHAPE;
  const int64_t tokens = static_cast<int64_t>(a.F) * a.T;
  // TMA coordinates and per-frame token offsets are 32-bit.
  if (tokens > INT32_MAX || static_cast<int64_t>(a.B) * a.H > (int64_t(1) << 24) ||
      static_cast<int64_t>(a.T) + gla::kTileTokens > INT32_MAX)
    return GLA_ERR_SHAPE;
  const int64_t elems = static_cast<int64_t>(a.B) * tokens * a.H * a.d;
  const int64_t units = static_cast<int64_t>(a.B) * a.F * a.H;
  if (elems > (int64_t(1) << 46) || units > INT32_MAX / 2) return GLA_ERR_SHAPE;
  if (elems > 0 && (a.q == nullptr || a.k == nullptr || a.v == nullptr || a.out == nullptr))
    return GLA_ERR_NULL;
  if (units > 0 && a.g == nullptr) return GLA_ERR_NULL;
  if (elems > 0 && (!aligned(a.q, 16) || !aligned(a.k, 16) || !aligned(a.v, 16) ||
                    !aligned(a.out, 16)))
    return GLA_ERR_ALIGN;
  if ((a.g && !aligned(a.g, 4)) || (a.s_in && !aligned(a.s_in, 4)) ||
      (a.s_out && !aligned(a.s_out, 4)))
    return GLA_ERR_ALIGN;
  return GLA_OK;
}

inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Launch as a programmatic dependent of the previous kernel in the stream:
// the grid may be scheduled before its predecessor finishes and must execute
// griddepcontrol.wait before reading anything the predecessor writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block,
                             size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The context a training forward saves for gla_backward_saved (d = 128):
// per unit the bf16 image of S_f^T (as the output kernel reads it), its bf16
// remainder (value rows 0..d-1) and S_f in fp32 ([d+1][d], as the scan writes
// them for the backward's query kernel), each region 256-byte aligned.
struct SavedLayout {
  int64_t image, image_lo, states, total;  // byte offsets, size
};
SavedLayout saved_layout(int64_t units) {
  constexpr int D = 128;
  SavedLayout l;
  const int64_t img = align256(units * static_cast<int64_t>(Geo<D>::kImageBytes));
  l.image = 0;
  l.image_lo = img;
  l.states = 2 * img;
  l.total = 2 * img + align256(units * static_cast<int64_t>(gla::IncCfg<D>::kPartialFloats) * 4);
  return l;
}

template <int D, bool kRope = false>
int run(const Args& a, const DeviceInfo& di, cudaEvent_t* ev,
        const FixedScratch* fixed = nullptr) {
  using G = Geo<D>;
  const int64_t units = static_cast<int64_t>(a.B) * a.F * a.H;
  const int tpu = (a.T + gla::kTileTokens - 1) / gla::kTileTokens;
  const int64_t W = units * tpu;
  const int32_t G1 = static_cast<int32_t>(W < di.sms ? W : di.sms);
  const int32_t G3 = G1;
  const gla::WorkPlan wp = W > 0 ? gla::WorkPlan::make(units, tpu, G1) : gla::WorkPlan{};

  const int64_t partial_bytes =
      W > 0 ? align256((units + G1) * static_cast<int64_t>(gla::IncCfg<D>::kPartialFloats) * 4) : 0;
  const int64_t image_bytes = W > 0 ? align256(units * static_cast<int64_t>(G::kImageBytes)) : 0;
  // rotary variant: the (cos, sin) table and the fp32 normaliser column per unit
  gla::RopeGeo rg{};
  int64_t table_pairs = 0;
  if (kRope && W > 0) {
    rg.dt = a.rope->dim_t;
    rg.dy = a.rope->dim_y;
    rg.dx = a.rope->dim_x;
    rg.grid_w = a.rope->grid_w;
    rg.rows = (a.T + rg.grid_w - 1) / rg.grid_w;
    rg.cols = a.T < rg.grid_w ? a.T : rg.grid_w;
    rg.frames = a.F;
    rg.frame_offset = a.rope->frame_offset;
    rg.sec_y = static_cast<int64_t>(a.F) * (rg.dt / 2);
    rg.sec_x = rg.sec_y + static_cast<int64_t>(rg.rows) * (rg.dy / 2);
    rg.sec_inc = rg.sec_x + static_cast<int64_t>(rg.cols) * (rg.dx / 2);
    table_pairs = rg.sec_inc + D;  // two increments per pair
    // token rows between consecutive rows of one ReLU thread (both kernels)
    static_assert(gla::IncCfg<D, true>::kReluWarps == gla::OutCfg<D, true>::kReluWarps,
                  "one row stride for the rotary kernels");
    rg.rpp = gla::IncCfg<D, true>::kReluWarps * 32 / Geo<D>::kChunksPerRow;
  }
  const int64_t table_bytes = align256(table_pairs * 8);
  const int64_t zvec_bytes = (kRope && W > 0) ? align256(units * static_cast<int64_t>(D) * 4) : 0;
  // single frame, plain layer: the increment kernel folds the scan step for
  // the units it owns whole; the scan runs over the split units alone
  // (a training forward writes every unit's state through the scan)
  const bool fold = !kRope && a.F == 1 && W > 0 && a.saved == nullptr;
  const SavedLayout sl = saved_layout(units);
  const int64_t ws_image_bytes = a.saved != nullptr ? 0 : image_bytes;
  const int64_t ws_bytes = partial_bytes + ws_image_bytes + table_bytes + zvec_bytes;

  CUtensorMap tm_q, tm_k, tm_v, tm_out;
  if (W > 0) {
    int st;
    if ((st = encode_map(&tm_q, a.q, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_k, a.k, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_v, a.v, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_out, a.out, D, a.H, a.T, a.F, a.B, 32)) != GLA_OK) return st;
  }

  uint8_t* ws = nullptr;
  if (fixed != nullptr) {
    if (static_cast<size_t>(ws_bytes) > fixed->bytes) return GLA_ERR_SCRATCH;
    ws = ws_bytes > 0 ? fixed->ptr : nullptr;
  } else {
    const int st = take_workspace(ws_bytes, a.stream, &ws);
    if (st != GLA_OK) return st;
  }
  float* partial = reinterpret_cast<float*>(ws);
  uint8_t* image = a.saved != nullptr ? a.saved + sl.image : (ws ? ws + partial_bytes : nullptr);
  float2* table = table_pairs > 0 ? reinterpret_cast<float2*>(ws + partial_bytes + ws_image_bytes)
                                  : nullptr;
  float* zvec = zvec_bytes > 0
                    ? reinterpret_cast<float*>(ws + partial_bytes + ws_image_bytes + table_bytes)
                    : nullptr;

  rg.table = reinterpret_cast<const float4*>(table);

  int status = GLA_OK;
  auto check = [&]() {
    if (cudaGetLastError() != cudaSuccess) status = GLA_ERR_LAUNCH;
  };
  auto record = [&](int i) {
    if (ev != nullptr && status == GLA_OK && cudaEventRecord(ev[i], a.stream) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
  };

  record(0);
  if (table_pairs > 0 && status == GLA_OK) {
    const int64_t blocks = (table_pairs + 255) / 256;
    gla::gla_rope_table_kernel<<<static_cast<unsigned>(blocks < 4 * di.sms ? blocks : 4 * di.sms),
                                 256, 0, a.stream>>>(table, rg,
                                                     std::log2(static_cast<double>(a.rope->theta)));
    check();
  }
  if (W > 0 && status == GLA_OK) {
    gla::IncParams ip{partial, wp, a.H, a.F, a.T, rg};
    if (fold) {
      ip.fold = 1;
      ip.gate = a.g;
      ip.state_in = a.s_in;
      ip.state_out = a.s_out;
      ip.image = image;
    }
    if (launch_dependent(gla::gla_increment_kernel<D, kRope>, G1, gla::IncCfg<D, kRope>::kThreads,
                         gla::IncCfg<D, kRope>::kSmemBytes, a.stream, tm_k, tm_v,
                         ip) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(1);
  // (b, h) pairs the scan covers: all, or with the fold the split units only
  const int32_t bh0 = fold ? wp.full_units() : 0;
  const int64_t nbh = static_cast<int64_t>(a.B) * a.H - bh0;
  if (status == GLA_OK && nbh > 0 && (a.F > 0 || a.s_out != nullptr)) {
    gla::ScanParams sp{partial, a.g, a.s_in, a.s_out, image, nullptr, wp, a.H, a.F, tpu, zvec};
    sp.bh0 = bh0;
    if (a.saved != nullptr) {  // the backward's inputs as well
      sp.states = reinterpret_cast<float*>(a.saved + sl.states);
      sp.image_lo = a.saved + sl.image_lo;
    }
    using SC1 = gla::ScanCfg<D, 1>;
    using SC3 = gla::ScanCfg<D, kScanStages>;
    const unsigned grid = static_cast<unsigned>(SC3::kGroups) * static_cast<unsigned>(nbh);
    const cudaError_t e =
        a.F <= 1 ? launch_dependent(gla::gla_scan_kernel<D, 1>, grid, SC1::kThreads,
                                    SC1::kSmemBytes, a.stream, sp)
                 : launch_dependent(gla::gla_scan_kernel<D, kScanStages>, grid, SC3::kThreads,
                                    SC3::kSmemBytes, a.stream, sp);
    if (e != cudaSuccess) status = GLA_ERR_LAUNCH;
    check();
  }
  record(2);
  if (W > 0 && status == GLA_OK) {
    gla::OutParams op{image, a.eps, wp, a.H, a.F, a.T, zvec, rg};
    if (launch_dependent(gla::gla_output_kernel<D, kRope>, G3, gla::OutCfg<D, kRope>::kThreads,
                         gla::OutCfg<D, kRope>::kSmemBytes, a.stream, tm_q, tm_out,
                         op) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(3);
  if (fixed == nullptr && ws != nullptr && cudaFreeAsync(ws, a.stream) != cudaSuccess) {
    cudaGetLastError();
    if (status == GLA_OK) status = GLA_ERR_LAUNCH;
  }
  return status;
}

// The frame-wise delta-rule variant: increment + Gram partials, the delta
// scan, the output kernel.
template <int D>
int run_gdn(const Args& a, const DeviceInfo& di, cudaEvent_t* ev) {
  using G = Geo<D>;
  using GC = gla::GdnScanCfg<D>;
  const int64_t units = static_cast<int64_t>(a.B) * a.F * a.H;
  const int tpu = (a.T + gla::kTileTokens - 1) / gla::kTileTokens;
  const int64_t W = units * tpu;
  const int32_t G1 = static_cast<int32_t>(W < di.sms ? W : di.sms);
  const gla::WorkPlan wp = W > 0 ? gla::WorkPlan::make(units, tpu, G1) : gla::WorkPlan{};
  const int64_t slots = units + G1;
  const int64_t partial_bytes =
      W > 0 ? align256(slots * static_cast<int64_t>(gla::IncCfg<D>::kPartialFloats) * 4) : 0;
  const int64_t mpartial_bytes = W > 0 ? align256(slots * static_cast<int64_t>(D) * D * 4) : 0;
  const int64_t image_bytes = W > 0 ? align256(units * static_cast<int64_t>(G::kImageBytes)) : 0;
  // d = 128: the tail units' Gram images (the tensor-core scan's A operands)
  const int32_t tail_units = W > 0 ? wp.units - wp.full_units() : 0;
  const int64_t mtail_bytes =
      D == 128 ? align256(static_cast<int64_t>(tail_units) * 2 * gla::GramImage<D>::kBytes) : 0;
  const int64_t ws_bytes = partial_bytes + mpartial_bytes + image_bytes + mtail_bytes;

  // state columns per scan block: as many blocks per (b, h) as fill the SMs
  // once, at least ceil((D + 1) / kMaxCols) and at most one per 8 columns
  const int64_t bh = static_cast<int64_t>(a.B) * a.H;
  // d = 128: the tensor-core scan (columns per block <= 48); else CUDA cores
  constexpr int kMaxCols = (D == 128) ? 48 : GC::kMaxCols;
  const int min_groups = (D + 1 + kMaxCols - 1) / kMaxCols;
  const int max_groups = (D + 1 + 7) / 8;
  int64_t want = bh > 0 ? di.sms / bh : 1;
  const int groups0 = static_cast<int>(want < min_groups ? min_groups
                                                         : (want > max_groups ? max_groups : want));
  const int cols = (D + 1 + groups0 - 1) / groups0;
  const int groups = (D + 1 + cols - 1) / cols;

  CUtensorMap tm_q, tm_k, tm_v, tm_out;
  if (W > 0) {
    int st;
    if ((st = encode_map(&tm_q, a.q, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_k, a.k, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_v, a.v, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_out, a.out, D, a.H, a.T, a.F, a.B, 32)) != GLA_OK) return st;
  }
  uint8_t* ws = nullptr;
  {
    const int st = take_workspace(ws_bytes, a.stream, &ws);
    if (st != GLA_OK) return st;
  }
  float* partial = W > 0 ? reinterpret_cast<float*>(ws) : nullptr;
  float* mpartial = W > 0 ? reinterpret_cast<float*>(ws + partial_bytes) : nullptr;
  uint8_t* image = W > 0 ? ws + partial_bytes + mpartial_bytes : nullptr;
  uint8_t* mtail = mtail_bytes > 0 ? ws + partial_bytes + mpartial_bytes + image_bytes : nullptr;

  int status = GLA_OK;
  auto check = [&]() {
    if (cudaGetLastError() != cudaSuccess) status = GLA_ERR_LAUNCH;
  };
  auto record = [&](int i) {
    if (ev != nullptr && status == GLA_OK && cudaEventRecord(ev[i], a.stream) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
  };
  record(0);
  if (W > 0 && status == GLA_OK) {
    gla::IncParams ip{partial, wp, a.H, a.F, a.T, gla::RopeGeo{}, mpartial};
    using IC = gla::IncCfg<D, false, true>;
    if (launch_dependent(gla::gla_increment_kernel<D, false, true>, G1, IC::kThreads,
                         IC::kSmemBytes, a.stream, tm_k, tm_v, ip) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  // the tail units' Gram partials -> one per unit
  if (tail_units > 0 && status == GLA_OK) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tail_units), 4);
    cfg.blockDim = dim3(256);
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if constexpr (D == 128) {
      // the tensor-core scan reads one Gram image and one dS partial per unit
      cfg.gridDim = dim3(static_cast<unsigned>(tail_units), gla::kGramParts + gla::kDsParts);
      e = cudaLaunchKernelEx(&cfg, gla::gla_gdn_tail_reduce_kernel<D>, partial,
                             static_cast<const float*>(mpartial), mtail, wp);
    } else {
      e = cudaLaunchKernelEx(&cfg, gla::gla_gram_reduce_kernel<D>, mpartial, wp);
    }
    if (e != cudaSuccess) status = GLA_ERR_LAUNCH;
    check();
  }
  record(1);
  if (status == GLA_OK && (a.F > 0 || a.s_out != nullptr)) {
    gla::GdnScanParams sp{partial, mpartial, mtail, a.g, a.beta, a.s_in, a.s_out, image, wp,
                          a.H, a.F, tpu, groups, cols};
    const unsigned grid = static_cast<unsigned>(groups) * static_cast<unsigned>(bh);
    cudaError_t e;
    if constexpr (D == 128)
      e = launch_dependent(gla::gla_gdn_scan_tc_kernel<128>, grid, gla::GdnTcCfg<128>::kThreads,
                           gla::GdnTcCfg<128>::kSmemBytes, a.stream, sp);
    else
      e = launch_dependent(gla::gla_gdn_scan_kernel<D>, grid, GC::kThreads, GC::kSmemBytes,
                           a.stream, sp);
    if (e != cudaSuccess) status = GLA_ERR_LAUNCH;
    check();
  }
  record(2);
  if (W > 0 && status == GLA_OK) {
    gla::OutParams op{image, a.eps, wp, a.H, a.F, a.T};
    if (launch_dependent(gla::gla_output_kernel<D>, G1, gla::OutCfg<D>::kThreads,
                         gla::OutCfg<D>::kSmemBytes, a.stream, tm_q, tm_out, op) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(3);
  if (ws != nullptr && cudaFreeAsync(ws, a.stream) != cudaSuccess) {
    cudaGetLastError();
    if (status == GLA_OK) status = GLA_ERR_LAUNCH;
  }
  return status;
}

int forward_impl(const Args& a, cudaEvent_t* ev) {
  int st = validate(a);
  if (st != GLA_OK) return st;
  if (a.rope != nullptr && (st = validate_rope(a.rope, a.d)) != GLA_OK) return st;
  if (a.beta != nullptr && !aligned(a.beta, 4)) return GLA_ERR_ALIGN;
  if (static_cast<int64_t>(a.B) * a.H == 0) return GLA_OK;  // nothing to compute or write
  DeviceInfo di;
  if ((st = device_setup(&di)) != GLA_OK) return st;
  if (a.beta != nullptr) {
    switch (a.d) {
      case 32: return run_gdn<32>(a, di, ev);
      case 64: return run_gdn<64>(a, di, ev);
      default: return run_gdn<128>(a, di, ev);
    }
  }
  if (a.rope != nullptr) {
    switch (a.d) {
      case 32: return run<32, true>(a, di, ev);
      case 64: return run<64, true>(a, di, ev);
      default: return run<128, true>(a, di, ev);
    }
  }
  switch (a.d) {
    case 32: return run<32>(a, di, ev);
    case 64: return run<64>(a, di, ev);
    default: return run<128>(a, di, ev);
  }
}

// One-time per-device lookup of g_gla_scratch's device address, made with
// that device current (the caller's current device).
int noalloc_setup(DeviceInfo* out) {
  int st = device_setup(out);
  if (st != GLA_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.scratch == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gla_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GLA_ERR_LAUNCH;
    }
    di.scratch = p;
  }
  *out = di;
  return GLA_OK;
}

int forward_noalloc_impl(const Args& a) {
  int st = validate(a);
  if (st != GLA_OK) return st;
  if (static_cast<int64_t>(a.B) * a.H == 0) return GLA_OK;
  DeviceInfo di;
  if ((st = noalloc_setup(&di)) != GLA_OK) return st;
  const FixedScratch fs{static_cast<uint8_t*>(di.scratch), kNoAllocScratchBytes};
  switch (a.d) {
    case 32: return run<32>(a, di, nullptr, &fs);
    case 64: return run<64>(a, di, nullptr, &fs);
    default: return run<128>(a, di, nullptr, &fs);
  }
}

struct BwdArgs {
  const void *q, *k, *v;
  const float* g;
  const float* s_in;
  const void* dout;
  const float* ds_out;
  void *dq, *dk, *dv;
  float* dg;
  float* ds_in;
  int B, H, F, T, d;
  float eps;
  cudaStream_t stream;
  const uint8_t* saved = nullptr;  // a training forward's context: no recompute
};

// Host-only checks of gla_backward's arguments; no CUDA call.
int validate_bwd(const BwdArgs& a) {
  if (a.d != 128) return GLA_ERR_UNSUPPORTED_D;
  Args f{a.q, a.k, a.v, a.g, a.s_in, nullptr, a.dq, a.B, a.H, a.F, a.T, a.d, a.eps, a.stream};
  int st = validate(f);
  if (st != GLA_OK) return st;
  const int64_t elems = static_cast<int64_t>(a.B) * a.F * a.T * a.H * a.d;
  const int64_t units = static_cast<int64_t>(a.B) * a.F * a.H;
  if (elems > 0 && (a.dout == nullptr || a.dk == nullptr || a.dv == nullptr)) return GLA_ERR_NULL;
  if (units > 0 && a.dg == nullptr) return GLA_ERR_NULL;
  if (elems > 0 && (!aligned(a.dout, 16) || !aligned(a.dk, 16) || !aligned(a.dv, 16)))
    return GLA_ERR_ALIGN;
  if ((a.dg && !aligned(a.dg, 4)) || (a.ds_out && !aligned(a.ds_out, 4)) ||
      (a.ds_in && !aligned(a.ds_in, 4)))
    return GLA_ERR_ALIGN;
  return GLA_OK;
}

// The six kernels of the backward pass (d = 128).  The workspace holds the
// partials (the recompute's increments, then the local state gradients L_f:
// the forward scan has finished reading the first before the query kernel
// writes the second), the bf16 images (S_f^T, then the hi part of G_f^T,
// likewise), the fp32 forward states S_f, the per-warp partial sums of da_f,
// the lo parts of the images (S_f^T, then G_f^T) and the fp32 normaliser rows
// G_f[:, d].
int run_backward(const BwdArgs& a, const DeviceInfo& di, cudaEvent_t* ev) {
  constexpr int D = 128;
  using G = Geo<D>;
  constexpr int PF = gla::IncCfg<D>::kPartialFloats;
  using RS = gla::ScanBwdCfg<D>;
  const int64_t units = static_cast<int64_t>(a.B) * a.F * a.H;
  const int tpu = (a.T + gla::kTileTokens - 1) / gla::kTileTokens;
  const int64_t W = units * tpu;
  const int32_t G1 = static_cast<int32_t>(W < di.sms ? W : di.sms);
  const gla::WorkPlan wp = W > 0 ? gla::WorkPlan::make(units, tpu, G1) : gla::WorkPlan{};

  const int64_t partial_bytes = W > 0 ? align256((units + G1) * static_cast<int64_t>(PF) * 4) : 0;
  const int64_t image_bytes = W > 0 ? align256(units * static_cast<int64_t>(G::kImageBytes)) : 0;
  const int64_t states_bytes = align256(units * static_cast<int64_t>(PF) * 4);
  const int64_t da_bytes = align256(units * static_cast<int64_t>(RS::kGroups) * 8 * 4);
  const int64_t gnorm_bytes = W > 0 ? align256(units * static_cast<int64_t>(D) * 4) : 0;
  const bool saved = a.saved != nullptr;
  // with a saved context the S_f images and states are read from it and the
  // G_f^T images go to the workspace (the caller's context is not written)
  const int64_t ws_bytes =
      partial_bytes + 2 * image_bytes + (saved ? 0 : states_bytes) + da_bytes + gnorm_bytes;

  CUtensorMap tm_q, tm_k, tm_v, tm_dout, tm_dq, tm_dk, tm_dv;
  if (W > 0) {
    int st;
    if ((st = encode_map(&tm_dout, a.dout, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK)
      return st;
    if ((st = encode_map(&tm_q, a.q, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_k, a.k, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    if ((st = encode_map(&tm_v, a.v, D, a.H, a.T, a.F, a.B, gla::kTileTokens)) != GLA_OK) return st;
    // gradient stores: 32 tokens x 32 features per warp and round (64-byte swizzle)
    if ((st = encode_map(&tm_dq, a.dq, D, a.H, a.T, a.F, a.B, 32, 32)) != GLA_OK) return st;
    if ((st = encode_map(&tm_dk, a.dk, D, a.H, a.T, a.F, a.B, 32, 32)) != GLA_OK) return st;
    if ((st = encode_map(&tm_dv, a.dv, D, a.H, a.T, a.F, a.B, 32, 32)) != GLA_OK) return st;
  }

  uint8_t* ws = nullptr;
  {
    const int st = take_workspace(ws_bytes, a.stream, &ws);
    if (st != GLA_OK) return st;
  }
  const int64_t ws_states = saved ? 0 : states_bytes;
  float* partial = W > 0 ? reinterpret_cast<float*>(ws) : nullptr;
  uint8_t* image = W > 0 ? ws + partial_bytes : nullptr;  // S_f^T (recompute), then G_f^T
  float* states = ws ? reinterpret_cast<float*>(ws + partial_bytes + image_bytes) : nullptr;
  float* da_part =
      ws ? reinterpret_cast<float*>(ws + partial_bytes + image_bytes + ws_states) : nullptr;
  uint8_t* image_lo = W > 0 ? ws + partial_bytes + image_bytes + ws_states + da_bytes : nullptr;
  float* gnorm = W > 0 ? reinterpret_cast<float*>(image_lo + image_bytes) : nullptr;
  // the query kernel's S_f inputs: the recompute's, or the saved context's
  const uint8_t* s_image = image;
  const uint8_t* s_image_lo = image_lo;
  const float* s_states = states;
  if (saved) {
    const SavedLayout sl = saved_layout(units);
    s_image = a.saved + sl.image;
    s_image_lo = a.saved + sl.image_lo;
    s_states = reinterpret_cast<const float*>(a.saved + sl.states);
    states = nullptr;
  }

  int status = GLA_OK;
  auto check = [&]() {
    if (cudaGetLastError() != cudaSuccess) status = GLA_ERR_LAUNCH;
  };
  auto record = [&](int i) {
    if (ev != nullptr && status == GLA_OK && cudaEventRecord(ev[i], a.stream) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
  };

  record(0);
  if (!saved && W > 0 && status == GLA_OK) {
    gla::IncParams ip{partial, wp, a.H, a.F};
    if (launch_dependent(gla::gla_increment_kernel<D>, G1, gla::IncCfg<D>::kThreads,
                         gla::IncCfg<D>::kSmemBytes, a.stream, tm_k, tm_v, ip) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(1);
  if (!saved && status == GLA_OK && a.F > 0) {
    gla::ScanParams sp{partial, a.g, a.s_in, nullptr, image, states, wp, a.H, a.F, tpu,
                       nullptr, image_lo};
    using SC1 = gla::ScanCfg<D, 1>;
    using SC3 = gla::ScanCfg<D, kScanStages>;
    const unsigned grid = static_cast<unsigned>(SC3::kGroups) * static_cast<unsigned>(a.B * a.H);
    const cudaError_t e =
        a.F <= 1 ? launch_dependent(gla::gla_scan_kernel<D, 1>, grid, SC1::kThreads,
                                    SC1::kSmemBytes, a.stream, sp)
                 : launch_dependent(gla::gla_scan_kernel<D, kScanStages>, grid, SC3::kThreads,
                                    SC3::kSmemBytes, a.stream, sp);
    if (e != cudaSuccess) status = GLA_ERR_LAUNCH;
    check();
  }
  record(2);
  if (W > 0 && status == GLA_OK) {
    gla::BwdQParams qp{s_image, s_image_lo, s_states, partial, a.eps, wp, a.H, a.F, a.T};
    if (launch_dependent(gla::gla_bwd_q_kernel<D>, G1, gla::BwdQCfg<D>::kThreads,
                         gla::BwdQCfg<D>::kSmemBytes, a.stream, tm_q, tm_dout, tm_dq,
                         qp) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(3);
  if (status == GLA_OK && (a.F > 0 || a.ds_in != nullptr)) {
    gla::ScanBwdParams rp{partial, a.g,   s_states, a.s_in, a.ds_out, a.ds_in, image,
                          image_lo, gnorm, da_part, wp,     a.H,    a.F,      tpu};
    const unsigned grid = static_cast<unsigned>(RS::kGroups) * static_cast<unsigned>(a.B * a.H);
    if (launch_dependent(gla::gla_scan_bwd_kernel<D>, grid, RS::kThreads, RS::kSmemBytes,
                         a.stream, rp) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(4);
  if (status == GLA_OK && units > 0) {
    const unsigned grid = static_cast<unsigned>((units + 255) / 256);
    if (launch_dependent(gla::gla_dgate_kernel<D>, grid, 256, 0, a.stream,
                         static_cast<const float*>(da_part), a.g, a.dg, units) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(5);
  if (W > 0 && status == GLA_OK) {
    gla::BwdKVParams kp{image, image_lo, gnorm, wp, a.H, a.F, a.T};
    if (launch_dependent(gla::gla_bwd_kv_kernel<D>, G1, gla::BwdKVCfg<D>::kThreads,
                         gla::BwdKVCfg<D>::kSmemBytes, a.stream, tm_k, tm_v, tm_dk, tm_dv,
                         kp) != cudaSuccess)
      status = GLA_ERR_LAUNCH;
    check();
  }
  record(6);
  if (ws != nullptr && cudaFreeAsync(ws, a.stream) != cudaSuccess) {
    cudaGetLastError();
    if (status == GLA_OK) status = GLA_ERR_LAUNCH;
  }
  return status;
}

int backward_impl(const BwdArgs& a, cudaEvent_t* ev) {
  int st = validate_bwd(a);
  if (st != GLA_OK) return st;
  if (static_cast<int64_t>(a.B) * a.H == 0) return GLA_OK;
  DeviceInfo di;
  if ((st = device_setup(&di)) != GLA_OK) return st;
  return run_backward(a, di, ev);
}

// The softmax anchor layer (d = 128).
// A rollout step of the anchor layer: the sink and window caches (see
// gla_softmax_anchor_step).  nullptr: a call over the whole sequence.
struct AnchorStep {
  const void *sink_k, *sink_v, *win_k, *win_v;
  int frame;
};

int anchor_impl(const void* q, const void* k, const void* v, const void* z, void* out, int B,
                int H, int F, int T, int d, int window, int n_sink, cudaStream_t stream,
                cudaEvent_t* ev, const AnchorStep* step = nullptr) {
  if (d != 128) return GLA_ERR_UNSUPPORTED_D;
  Args chk{q, k, v, nullptr, nullptr, nullptr, out, B, H, F, T, d, 0.f, stream};
  const int64_t units0 = static_cast<int64_t>(B) * F * H;
  static const float kNone = 0.f;  // the validator wants gate logits when units > 0
  chk.g = units0 > 0 ? &kNone : nullptr;
  int st = validate(chk);
  if (st != GLA_OK) return st;
  if (window < 1 || n_sink < 0) return GLA_ERR_SHAPE;
  if (z != nullptr && !aligned(z, 16)) return GLA_ERR_ALIGN;
  // rollout step: the frames of the window before this one come from the
  // window cache, the sink tokens that precede the window from the sink cache
  int win_frames = 0, sinks = 0;
  if (step != nullptr) {
    if (step->frame < 0) return GLA_ERR_SHAPE;
    win_frames = step->frame < window - 1 ? step->frame : window - 1;
    const int64_t w_lo = static_cast<int64_t>(step->frame - win_frames) * T;
    sinks = static_cast<int>(n_sink < w_lo ? n_sink : w_lo);
    if (static_cast<int64_t>(B) * H * T > 0) {
      if (win_frames > 0 && (step->win_k == nullptr || step->win_v == nullptr))
        return GLA_ERR_NULL;
      if (sinks > 0 && (step->sink_k == nullptr || step->sink_v == nullptr)) return GLA_ERR_NULL;
      if ((win_frames > 0 && (!aligned(step->win_k, 16) || !aligned(step->win_v, 16))) ||
          (sinks > 0 && (!aligned(step->sink_k, 16) || !aligned(step->sink_v, 16))))
        return GLA_ERR_ALIGN;
    }
  }
  const int tpf = (T + gla::kTileTokens - 1) / gla::kTileTokens;
  const int64_t units = units0 * tpf;
  if (units > INT32_MAX) return GLA_ERR_SHAPE;
  if (units == 0) return GLA_OK;
  DeviceInfo di;
  if ((st = device_setup(&di)) != GLA_OK) return st;
  CUtensorMap tm_q, tm_k, tm_v, tm_z, tm_out;
  if ((st = encode_map(&tm_q, q, d, H, T, F, B, gla::kTileTokens)) != GLA_OK) return st;
  if ((st = encode_map(&tm_k, k, d, H, T, F, B, gla::kTileTokens)) != GLA_OK) return st;
  if ((st = encode_map(&tm_v, v, d, H, T, F, B, gla::kTileTokens)) != GLA_OK) return st;
  if ((st = encode_map(&tm_z, z != nullptr ? z : q, d, H, T, F, B, gla::kTileTokens)) != GLA_OK)
    return st;
  if ((st = encode_map(&tm_out, out, d, H, T, F, B, 32)) != GLA_OK) return st;
  gla::AnchorCaches caches;  // a whole-sequence call never reads them
  caches.ks = caches.vs = caches.kw = caches.vw = tm_k;
  if (step != nullptr) {
    if (sinks > 0 &&
        ((st = encode_map(&caches.ks, step->sink_k, d, H, n_sink, 1, B, gla::kTileTokens)) !=
             GLA_OK ||
         (st = encode_map(&caches.vs, step->sink_v, d, H, n_sink, 1, B, gla::kTileTokens)) !=
             GLA_OK))
      return st;
    if (win_frames > 0 &&
        ((st = encode_map(&caches.kw, step->win_k, d, H, T, win_frames, B, gla::kTileTokens)) !=
             GLA_OK ||
         (st = encode_map(&caches.vw, step->win_v, d, H, T, win_frames, B, gla::kTileTokens)) !=
             GLA_OK))
      return st;
  }
  gla::AnchorParams ap{H,
                       F,
                       T,
                       window,
                       n_sink,
                       static_cast<int>(units),
                       static_cast<float>(1.4426950408889634 / std::sqrt(128.0)),
                       z != nullptr,
                       step != nullptr,
                       step != nullptr ? step->frame : 0};
  const int grid = static_cast<int>(units < di.sms ? units : di.sms);
  int status = GLA_OK;
  if (ev != nullptr && cudaEventRecord(ev[0], stream) != cudaSuccess) return GLA_ERR_LAUNCH;
  gla::gla_softmax_anchor_kernel<128>
      <<<grid, gla::AnchorCfg<128>::kThreads, gla::AnchorCfg<128>::kSmemBytes, stream>>>(
          tm_q, tm_k, tm_v, tm_z, tm_out, caches, ap);
  if (cudaGetLastError() != cudaSuccess) status = GLA_ERR_LAUNCH;
  if (ev != nullptr && status == GLA_OK && cudaEventRecord(ev[1], stream) != cudaSuccess)
    status = GLA_ERR_LAUNCH;
  return status;
}

}  // namespace

extern "C" {

int gla_forward(const void* q, const void* k, const void* v, const float* gate_logits,
                const float* state_in, float* state_out, void* out, int B, int H, int frames,
                int tokens_per_frame, int d, float eps, cudaStream_t stream) {
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream};
  return forward_impl(a, nullptr);
}

int gla_forward_timed(const void* q, const void* k, const void* v, const float* gate_logits,
                      const float* state_in, float* state_out, void* out, int B, int H, int frames,
                      int tokens_per_frame, int d, float eps, cudaStream_t stream,
                      cudaEvent_t* events) {
  if (events == nullptr) return GLA_ERR_NULL;
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream};
  return forward_impl(a, events);
}

int gla_forward_noalloc(const void* q, const void* k, const void* v, const float* gate_logits,
                        const float* state_in, float* state_out, void* out, int B, int H,
                        int frames, int tokens_per_frame, int d, float eps, cudaStream_t stream) {
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream};
  return forward_noalloc_impl(a);
}

size_t gla_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int gla_softmax_anchor(const void* q, const void* k, const void* v, const void* gate_z,
                       void* out, int B, int H, int frames, int tokens_per_frame, int d,
                       int window_frames, int n_sink, cudaStream_t stream) {
  return anchor_impl(q, k, v, gate_z, out, B, H, frames, tokens_per_frame, d, window_frames,
                     n_sink, stream, nullptr);
}

int gla_softmax_anchor_timed(const void* q, const void* k, const void* v, const void* gate_z,
                             void* out, int B, int H, int frames, int tokens_per_frame, int d,
                             int window_frames, int n_sink, cudaStream_t stream,
                             cudaEvent_t* events) {
  if (events == nullptr) return GLA_ERR_NULL;
  return anchor_impl(q, k, v, gate_z, out, B, H, frames, tokens_per_frame, d, window_frames,
                     n_sink, stream, events);
}

int gla_softmax_anchor_step(const void* q, const void* k, const void* v, const void* gate_z,
                            const void* sink_k, const void* sink_v, const void* win_k,
                            const void* win_v, void* out, int B, int H, int tokens_per_frame,
                            int d, int frame, int window_frames, int n_sink,
                            cudaStream_t stream) {
  const AnchorStep st{sink_k, sink_v, win_k, win_v, frame};
  return anchor_impl(q, k, v, gate_z, out, B, H, 1, tokens_per_frame, d, window_frames, n_sink,
                     stream, nullptr, &st);
}

int gla_forward_gdn(const void* q, const void* k, const void* v, const float* gate_logits,
                    const float* beta_logits, const float* state_in, float* state_out, void* out,
                    int B, int H, int frames, int tokens_per_frame, int d, float eps,
                    cudaStream_t stream) {
  if (static_cast<int64_t>(B) * frames * H > 0 && beta_logits == nullptr) return GLA_ERR_NULL;
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream, nullptr, beta_logits};
  static const float kNone = 0.f;  // marks the variant when there are no units
  if (a.beta == nullptr) a.beta = &kNone;
  return forward_impl(a, nullptr);
}

int gla_forward_gdn_timed(const void* q, const void* k, const void* v, const float* gate_logits,
                          const float* beta_logits, const float* state_in, float* state_out,
                          void* out, int B, int H, int frames, int tokens_per_frame, int d,
                          float eps, cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr) return GLA_ERR_NULL;
  if (static_cast<int64_t>(B) * frames * H > 0 && beta_logits == nullptr) return GLA_ERR_NULL;
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream, nullptr, beta_logits};
  static const float kNone = 0.f;
  if (a.beta == nullptr) a.beta = &kNone;
  return forward_impl(a, events);
}

int gla_forward_rope(const void* q, const void* k, const void* v, const float* gate_logits,
                     const float* state_in, float* state_out, void* out, int B, int H, int frames,
                     int tokens_per_frame, int d, float eps, const gla_rope_config* rope,
                     cudaStream_t stream) {
  if (rope == nullptr) return GLA_ERR_NULL;
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream, rope};
  return forward_impl(a, nullptr);
}

int gla_forward_rope_timed(const void* q, const void* k, const void* v, const float* gate_logits,
                           const float* state_in, float* state_out, void* out, int B, int H,
                           int frames, int tokens_per_frame, int d, float eps,
                           const gla_rope_config* rope, cudaStream_t stream, cudaEvent_t* events) {
  if (rope == nullptr || events == nullptr) return GLA_ERR_NULL;
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream, rope};
  return forward_impl(a, events);
}

int gla_backward(const void* q, const void* k, const void* v, const float* gate_logits,
                 const float* state_in, const void* dout, const float* dstate_out, void* dq,
                 void* dk, void* dv, float* dgate_logits, float* dstate_in, int B, int H,
                 int frames, int tokens_per_frame, int d, float eps, cudaStream_t stream) {
  BwdArgs a{q,  k,  v,  gate_logits, state_in, dout, dstate_out, dq, dk,     dv,
            dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps, stream};
  return backward_impl(a, nullptr);
}

int gla_backward_timed(const void* q, const void* k, const void* v, const float* gate_logits,
                       const float* state_in, const void* dout, const float* dstate_out, void* dq,
                       void* dk, void* dv, float* dgate_logits, float* dstate_in, int B, int H,
                       int frames, int tokens_per_frame, int d, float eps, cudaStream_t stream,
                       cudaEvent_t* events) {
  if (events == nullptr) return GLA_ERR_NULL;
  BwdArgs a{q,  k,  v,  gate_logits, state_in, dout, dstate_out, dq, dk,     dv,
            dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps, stream};
  return backward_impl(a, events);
}

size_t gla_saved_bytes(int B, int H, int frames, int tokens_per_frame, int d) {
  if (d != 128 || B < 0 || H < 0 || frames < 0 || tokens_per_frame < 0) return 0;
  return static_cast<size_t>(saved_layout(static_cast<int64_t>(B) * frames * H).total);
}

int gla_forward_train(const void* q, const void* k, const void* v, const float* gate_logits,
                      const float* state_in, float* state_out, void* out, void* saved, int B,
                      int H, int frames, int tokens_per_frame, int d, float eps,
                      cudaStream_t stream) {
  Args a{q, k, v, gate_logits, state_in, state_out, out, B, H, frames, tokens_per_frame, d, eps,
         stream};
  int st = validate(a);
  if (st != GLA_OK) return st;
  if (d != 128) return GLA_ERR_UNSUPPORTED_D;
  if (static_cast<int64_t>(B) * frames * H > 0 && saved == nullptr) return GLA_ERR_NULL;
  if (!aligned(saved, 256)) return GLA_ERR_ALIGN;
  a.saved = static_cast<uint8_t*>(saved);
  return forward_impl(a, nullptr);
}

namespace {
int backward_saved(const BwdArgs& a, cudaEvent_t* ev) {
  int st = validate_bwd(a);
  if (st != GLA_OK) return st;
  if (static_cast<int64_t>(a.B) * a.F * a.H > 0 && a.saved == nullptr) return GLA_ERR_NULL;
  if (!aligned(a.saved, 256)) return GLA_ERR_ALIGN;
  return backward_impl(a, ev);
}
}  // namespace

int gla_backward_saved(const void* q, const void* k, const void* v, const float* gate_logits,
                       const float* state_in, const void* saved, const void* dout,
                       const float* dstate_out, void* dq, void* dk, void* dv, float* dgate_logits,
                       float* dstate_in, int B, int H, int frames, int tokens_per_frame, int d,
                       float eps, cudaStream_t stream) {
  BwdArgs a{q,  k,  v,  gate_logits, state_in, dout, dstate_out, dq, dk,     dv,
            dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps, stream,
            static_cast<const uint8_t*>(saved)};
  return backward_saved(a, nullptr);
}

int gla_backward_saved_timed(const void* q, const void* k, const void* v,
                             const float* gate_logits, const float* state_in, const void* saved,
                             const void* dout, const float* dstate_out, void* dq, void* dk,
                             void* dv, float* dgate_logits, float* dstate_in, int B, int H,
                             int frames, int tokens_per_frame, int d, float eps,
                             cudaStream_t stream, cudaEvent_t* events) {
  if (events == nullptr) return GLA_ERR_NULL;
  BwdArgs a{q,  k,  v,  gate_logits, state_in, dout, dstate_out, dq, dk,     dv,
            dgate_logits, dstate_in, B, H, frames, tokens_per_frame, d, eps, stream,
            static_cast<const uint8_t*>(saved)};
  return backward_saved(a, events);
}

int gla_trim_workspace(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GLA_ERR_DEVICE;
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    pool = g_pool[dev];
  }
  if (pool == nullptr) return GLA_OK;
  return cudaMemPoolTrimTo(pool, 0) == cudaSuccess ? GLA_OK : GLA_ERR_LAUNCH;
}

int gla_set_workspace_retention(unsigned long long bytes) {
  cudaMemPool_t pool = workspace_pool();
  if (pool == nullptr) return GLA_ERR_DEVICE;
  uint64_t keep = bytes;
  if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
    cudaGetLastError();
    return GLA_ERR_LAUNCH;
  }
  return GLA_OK;
}

int gla_set_wait_limit_ns(unsigned long long ns) {
  const uint64_t v = ns == 0 ? gla::kWaitLimitDefaultNs : static_cast<uint64_t>(ns);
  if (cudaMemcpyToSymbol(gla::g_gla_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return GLA_ERR_LAUNCH;
  }
  return GLA_OK;
}

int gla_inject_stall(long long tile) {
  const long long v = tile < 0 ? -1 : tile;
  if (cudaMemcpyToSymbol(gla::g_gla_stall_tile, &v, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return GLA_ERR_LAUNCH;
  }
  return GLA_OK;
}

int gla_inject_alloc_failure(int count) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_fail_allocs = count > 0 ? count : 0;
  return GLA_OK;
}

const char* gla_error_string(int status) {
  switch (status) {
    case GLA_OK: return "ok";
    case GLA_ERR_NULL: return "a required pointer is NULL";
    case GLA_ERR_ALIGN: return "a pointer is not aligned (q, k, v, out: 16 bytes; others: 4)";
    case GLA_ERR_SHAPE: return "negative or too large size";
    case GLA_ERR_UNSUPPORTED_D:
      return "head dim must be 32, 64 or 128 (gla_backward: 128)";
    case GLA_ERR_ALLOC: return "workspace allocation failed";
    case GLA_ERR_LAUNCH: return "CUDA runtime call or kernel launch failed";
    case GLA_ERR_DEVICE: return "no CUDA device of compute capability 10.x";
    case GLA_ERR_SCRATCH:
      return "problem needs more scratch than gla_forward_noalloc's fixed 32 MiB buffer";
    case GLA_ERR_ROPE:
      return "invalid rotary configuration (blocks: multiples of 8 summing to d; grid_w >= 1; "
             "0 <= frame_offset <= 2^24; theta > 0 and finite)";
    default: return "unknown status";
  }
}

int gla_device_fault(cudaStream_t stream, unsigned int* code) {
  if (code == nullptr) return GLA_ERR_NULL;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GLA_ERR_LAUNCH;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, gla::g_gla_fault, sizeof(v)) != cudaSuccess) return GLA_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(gla::g_gla_fault, &zero, sizeof(zero)) != cudaSuccess)
    return GLA_ERR_LAUNCH;
  *code = v;
  return GLA_OK;
}

int gla_version(void) { return 100; }

}  // extern "C"
