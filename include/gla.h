/*
 * gla.h -- C ABI of the B200 (sm_100a) gated linear attention library.
 *
 * Operation (block-causal gated linear attention, one latent video frame per
 * block).  The SANA-Video pages describe the layer's structure: gated linear
 * attention is the O(N) mixer of the hybrid DiT (SANA-Video 2.0 project page,
 * "Hybrid Linear-Softmax Attention"); the state is a fixed-size D x D matrix
 * to which each block adds its own key-value contribution, cached between
 * blocks (SANA-Video ICLR 2026 oral talk, block KV cache segment); decay gates
 * on the recurrent state stop the drift of plain cumulative linear attention
 * and the attention is applied frame-wise (SANA-WM paper analysis, method
 * components).  This library fixes the formulas as follows, per batch entry b
 * and head h, frames f = 0..frames-1, tokens t of frame f:
 *
 *   phi(x) = max(x, 0)
 *   a_f    = 1 / (1 + exp(-gate_logits[b, f, h]))
 *   S_f    = a_f * S_{f-1} + phi(K_f)^T [V_f | 1]      (d x (d+1), fp32; S_{-1} = state_in)
 *   out_t  = (phi(q_t) S_f[:, :d]) / (phi(q_t) S_f[:, d] + eps)
 *   state_out = S_{frames-1}
 *
 * Queries of frame f read S_f: attention is bidirectional inside a frame and
 * causal across frames.  A long sequence can be streamed through several
 * calls by passing one call's state_out as the next call's state_in; the
 * result equals one call over all frames up to fp32 rounding.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller; the library keeps no reference after the call.
 *   - Work is enqueued on `stream` and the call returns without waiting.
 *     Errors found before launch are returned; faults inside the kernels
 *     surface at the caller's next synchronisation, and bounded waits that
 *     gave up are reported by gla_device_fault().
 *   - Supported head dims: d in {32, 64, 128}.  B, H, frames,
 *     tokens_per_frame may be 0 (nothing to attend; see gla_forward).
 *   - Requires a compute capability 10.0 device (B200, sm_100a).
 */
#ifndef GLA_H_
#define GLA_H_

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
typedef enum {
  GLA_OK = 0,
  GLA_ERR_NULL = 1,            /* a required pointer is NULL */
  GLA_ERR_ALIGN = 2,           /* a pointer violates its alignment rule */
  GLA_ERR_SHAPE = 3,           /* negative or too-large size */
  GLA_ERR_UNSUPPORTED_D = 4,   /* d not in {32, 64, 128} */
  GLA_ERR_ALLOC = 5,           /* stream-ordered workspace allocation failed */
  GLA_ERR_LAUNCH = 6,          /* a CUDA runtime call or kernel launch failed */
  GLA_ERR_DEVICE = 7,          /* no CUDA device, or not compute capability 10.x */
  GLA_ERR_SCRATCH = 8,         /* gla_forward_noalloc: problem exceeds the fixed scratch */
  GLA_ERR_ROPE = 9             /* gla_forward_rope: invalid rotary configuration */
} gla_status;

/*
 * gla_forward -- one block-causal gated linear attention layer call.
 *
 * Arguments (device pointers unless stated):
 *   q, k, v      bf16 [B, frames * tokens_per_frame, H, d], contiguous; token
 *                n = f * tokens_per_frame + t.  16-byte aligned.
 *   gate_logits  fp32 [B, frames, H]; a = sigmoid(logit).  +inf gives a = 1,
 *                -inf gives a = 0.  4-byte aligned.  Must not be NULL when
 *                B * H * frames > 0.
 *   state_in     fp32 [B, H, d, d + 1] (row i = key feature, column d = the
 *                normaliser); NULL means the zero state.  4-byte aligned.
 *   state_out    fp32 [B, H, d, d + 1]; NULL means "not written".  May be the
 *                same pointer as state_in (updated in place).
 *   out          bf16 [B, frames * tokens_per_frame, H, d], 16-byte aligned,
 *                rounded to nearest even.  Must not overlap q, k, v.
 *   B, H, frames, tokens_per_frame   sizes, each >= 0.  frames == 0 copies
 *                state_in to state_out; tokens_per_frame == 0 applies only
 *                the decays to the state.
 *   d            head dim: 32, 64 or 128.
 *   eps          added to the normaliser before the division.
 *   stream       CUDA stream for all work (0 = legacy default stream).
 *
 * Memory: takes a workspace of about (B*H*frames*6 + #SMs*4) * (d+1)*d bytes
 * (per-frame fp32 state increments and bf16 prefix states) from the
 * library's stream-ordered memory pool on `stream` and frees it on the same
 * stream.  The pool (one per device, created at the first call) keeps freed
 * memory mapped for later calls (gla_set_workspace_retention bounds that);
 * gla_trim_workspace() returns it.
 * Returns GLA_OK or a gla_status code; on error nothing was enqueued, except
 * GLA_ERR_LAUNCH, after which part of the work may have been enqueued.
 */
int gla_forward(const void* q, const void* k, const void* v,
                const float* gate_logits,
                const float* state_in, float* state_out,
                void* out,
                int B, int H, int frames, int tokens_per_frame, int d,
                float eps, cudaStream_t stream);

/*
 * gla_forward_timed -- gla_forward that also records four caller-created CUDA
 * events on `stream`: events[0] before the state-increment kernel, events[1]
 * after it, events[2] after the gated scan, events[3] after the output
 * kernel.  Used to time each kernel in place; the computation is identical.
 * `events` is a host array of 4 cudaEvent_t.
 */
int gla_forward_timed(const void* q, const void* k, const void* v,
                      const float* gate_logits,
                      const float* state_in, float* state_out,
                      void* out,
                      int B, int H, int frames, int tokens_per_frame, int d,
                      float eps, cudaStream_t stream, cudaEvent_t* events);

/*
 * gla_forward_noalloc -- gla_forward that allocates no device memory.
 *
 * No counterpart in the paper: this is a deployment variant.  Some callers
 * cannot allocate device memory while they run the layer: a serving process
 * whose own allocator reserves all free HBM at start-up (so a library
 * cudaMallocAsync fails or fragments that reserve), or a per-frame streaming
 * loop that must not enter the CUDA allocator, whose calls can block and
 * whose failures are hard to recover from mid-stream.  This entry point takes
 * the same arguments and computes the same result as gla_forward, with its
 * workspace in a fixed 32 MiB device array inside the library instead.
 *
 *   - Limit: the workspace must fit in 32 MiB (gla_noalloc_scratch_bytes()),
 *     i.e. about (B*H*frames*6 + #SMs*4)*(d+1)*d bytes <= 32 MiB.  At d = 128
 *     on a 148-SM B200 that is up to 240 (batch, frame, head) units per call,
 *     e.g. the one-frame streaming step of 8 sequences x 24 heads.  Larger
 *     problems return GLA_ERR_SCRATCH and nothing is enqueued.
 *   - The array exists on every device that loads the library, until exit.
 *   - The first call on each device performs a one-time set-up (it looks up
 *     the array's device address with that device current, and sets kernel
 *     attributes); make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Nothing in it needs to start at zero: every byte the kernels read was
 *     written earlier in the same call.  Calls that overlap on the GPU (for
 *     example on two streams at once) race on the array and give wrong
 *     results: serialise them.
 *   - Never calls cudaMalloc, cudaMallocAsync, cudaFree or any allocating
 *     routine.  Returns the gla_forward codes plus GLA_ERR_SCRATCH.
 */
int gla_forward_noalloc(const void* q, const void* k, const void* v,
                        const float* gate_logits,
                        const float* state_in, float* state_out,
                        void* out,
                        int B, int H, int frames, int tokens_per_frame, int d,
                        float eps, cudaStream_t stream);

/* Size in bytes of gla_forward_noalloc's fixed scratch array.  Host only. */
size_t gla_noalloc_scratch_bytes(void);

/*
 * gla_softmax_anchor -- the softmax anchor layer with attention sinks and a
 * local window of frames (d = 128 only).
 *
 * The SANA-Video 2.0 pages interleave gated-softmax anchors with the linear
 * layers (one in four); the SANA-WM pages add attention-sink tokens and local
 * temporal windows to the softmax layers so that their memory and per-chunk
 * latency stay constant over long rollouts.  No formula is printed; this
 * library reads it, per (b, h), frames f of tokens_per_frame tokens, as:
 *   keys of the queries of frame f = all tokens of frames
 *       max(0, f - window_frames + 1) .. f, plus the first n_sink tokens of
 *       the sequence that precede that window (never a later frame)
 *   out_t = sigmoid(gate_z_t) * sum_s softmax_s(q_t . k_s / sqrt(d)) v_s
 * Arguments: q, k, v, out bf16 [B, frames * tokens_per_frame, H, d]
 * (16-byte aligned, out not overlapping the inputs); gate_z bf16 of the same
 * shape or NULL (no gate); window_frames >= 1; n_sink >= 0.  No workspace.
 * Returns the gla_forward codes (GLA_ERR_SHAPE for window_frames < 1 or
 * n_sink < 0).
 * Precision: scores and row sums in fp32; the softmax weights enter P V
 * rounded to bf16 (some exponentials by a polynomial of relative error
 * 7.5e-5); out is rounded once to bf16.  Keys past a frame's end are masked;
 * a query always sees its own frame, so every row has at least one key.
 */
int gla_softmax_anchor(const void* q, const void* k, const void* v, const void* gate_z,
                       void* out, int B, int H, int frames, int tokens_per_frame, int d,
                       int window_frames, int n_sink, cudaStream_t stream);

/* gla_softmax_anchor with events[0] / events[1] recorded around the kernel. */
int gla_softmax_anchor_timed(const void* q, const void* k, const void* v, const void* gate_z,
                             void* out, int B, int H, int frames, int tokens_per_frame, int d,
                             int window_frames, int n_sink, cudaStream_t stream,
                             cudaEvent_t* events);

/*
 * gla_softmax_anchor_step -- the softmax anchor layer for one new frame of a
 * rollout, from cached keys and values.
 *
 * The SANA-WM pages (method components) give the softmax layers attention
 * sinks and a local window of frames so that memory and per-chunk latency
 * stay constant over a long rollout: a new frame needs only the sink tokens
 * and the window's earlier frames, not the whole sequence.  This call computes
 * the output of frame `frame` of the sequence exactly as gla_softmax_anchor
 * over the whole sequence would (the same key tiles in the same order, so the
 * result is the same bit for bit):
 *   q, k, v, gate_z, out   bf16 [B, T, H, d], the new frame (gate_z may be NULL)
 *   sink_k, sink_v         bf16 [B, n_sink, H, d]: the first n_sink tokens of the
 *                          sequence.  Only the min(n_sink, w_lo * T) of them
 *                          that precede the window are read, w_lo =
 *                          max(0, frame - window_frames + 1); NULL allowed when
 *                          that is 0.
 *   win_k, win_v           bf16 [B, nw * T, H, d]: the window's earlier frames
 *                          w_lo .. frame - 1, oldest first, nw = min(frame,
 *                          window_frames - 1); NULL allowed when nw = 0.
 *   frame >= 0, window_frames >= 1, n_sink >= 0, d = 128; T = tokens_per_frame.
 * The caller keeps the caches (a copy of the first n_sink keys and values and
 * of the last window_frames - 1 frames).  All pointers 16-byte aligned device
 * pointers.  Returns the gla_softmax_anchor codes.
 */
int gla_softmax_anchor_step(const void* q, const void* k, const void* v, const void* gate_z,
                            const void* sink_k, const void* sink_v, const void* win_k,
                            const void* win_v, void* out, int B, int H, int tokens_per_frame,
                            int d, int frame, int window_frames, int n_sink,
                            cudaStream_t stream);

/*
 * gla_forward_gdn -- the frame-wise gated delta-rule variant (Gated DeltaNet).
 *
 * The SANA-WM pages (paper analysis: abstract, method components) describe
 * the layer as frame-wise Gated DeltaNet: the SANA-Video linear attention
 * whose recurrent state gets decay gates and delta-rule corrections, with
 * keys scaled by 1/sqrt(D S).  No formula is printed; this library reads it
 * as the layer above with the frame's write made a delta rule:
 *   a_f = sigmoid(gate_logits[b, f, h]),  beta_f = sigmoid(beta_logits[b, f, h])
 *   S_f = a_f S_{f-1} + beta_f phi(K_f)^T ([V_f | 1] - a_f phi(K_f) S_{f-1})
 *   out_t = (phi(q_t) S_f[:, :d]) / (phi(q_t) S_f[:, d] + eps)
 * (the frame's keys read what the decayed state holds for them and write the
 * difference).  The key scale is the caller's: the recurrence contracts when
 * beta_f ||phi(K_f)^T phi(K_f)|| < 2, e.g. k ~ N(0, 1/(d T)).
 * Arguments as gla_forward plus beta_logits fp32 [B, frames, H] (4-byte
 * aligned; must not be NULL when B * H * frames > 0).  Workspace: as
 * gla_forward plus 4 d^2 bytes per (batch, frame, head) and per SM (at
 * d = 128 up to another 4 d^2 bytes per SM: the Gram matrices of the units
 * that the tile schedule splits over several SMs).
 */
int gla_forward_gdn(const void* q, const void* k, const void* v,
                    const float* gate_logits, const float* beta_logits,
                    const float* state_in, float* state_out,
                    void* out,
                    int B, int H, int frames, int tokens_per_frame, int d,
                    float eps, cudaStream_t stream);

/* gla_forward_gdn with four events recorded as in gla_forward_timed. */
int gla_forward_gdn_timed(const void* q, const void* k, const void* v,
                          const float* gate_logits, const float* beta_logits,
                          const float* state_in, float* state_out,
                          void* out,
                          int B, int H, int frames, int tokens_per_frame, int d,
                          float eps, cudaStream_t stream, cudaEvent_t* events);

/*
 * Rotary position embedding of gla_forward_rope.  The SANA-Video ICLR 2026
 * talk (temporal modelling segment) adds a 3D RoPE to the linear attention
 * without a formula; this library reads it in the RoFormer form for linear
 * attention.  Token t of frame f sits at
 *     (p_t, p_y, p_x) = (frame_offset + f, t / grid_w, t % grid_w);
 * the head dim is split into feature blocks [dim_t | dim_y | dim_x], and pair
 * j (features 2j, 2j+1 of a block of n features) turns by the angle
 * p_axis * theta^(-2j/n).  With R_t the rotation of token t:
 *     S_f[:, :d] = a_f S_{f-1}[:, :d] + (R phi(K_f))^T V_f
 *     S_f[:, d]  = a_f S_{f-1}[:, d]  + phi(K_f)^T 1          (not rotated)
 *     out_t = (R_t phi(q_t)) S_f[:, :d] / (phi(q_t) S_f[:, d] + eps)
 * The state keeps the rotated keys: a stream of calls passes state_out on as
 * state_in and advances frame_offset by the frames already processed.
 */
typedef struct {
  int grid_w;        /* tokens per latent row, >= 1 (80 for a 46 x 80 grid) */
  int frame_offset;  /* temporal position of the call's first frame, 0 .. 2^24 */
  int dim_t;         /* feature blocks: multiples of 8 (0 allowed), */
  int dim_y;         /*   dim_t + dim_y + dim_x == d              */
  int dim_x;
  float theta;       /* frequency base, > 0 and finite (e.g. 10000) */
} gla_rope_config;

/*
 * gla_forward_rope -- gla_forward with the rotary position embedding above
 * fused into the loads of the two tensor-core kernels.  Arguments as
 * gla_forward, plus `rope` (host pointer, read during the call only).
 * Returns GLA_ERR_NULL if rope is NULL and GLA_ERR_ROPE for an invalid
 * configuration (nothing enqueued); otherwise as gla_forward.  The workspace
 * adds a (cos, sin) table of 8 * (frames*dim_t/2 + rows*dim_y/2 +
 * min(T, grid_w)*dim_x/2) bytes (rows = ceil(T / grid_w)) and 4*d bytes per
 * (batch, frame, head).
 */
int gla_forward_rope(const void* q, const void* k, const void* v,
                     const float* gate_logits,
                     const float* state_in, float* state_out,
                     void* out,
                     int B, int H, int frames, int tokens_per_frame, int d,
                     float eps, const gla_rope_config* rope, cudaStream_t stream);

/* gla_forward_rope with four events recorded as in gla_forward_timed (the
 * table kernel counts with the state-increment kernel). */
int gla_forward_rope_timed(const void* q, const void* k, const void* v,
                           const float* gate_logits,
                           const float* state_in, float* state_out,
                           void* out,
                           int B, int H, int frames, int tokens_per_frame, int d,
                           float eps, const gla_rope_config* rope, cudaStream_t stream,
                           cudaEvent_t* events);

/*
 * gla_backward -- gradients of one gla_forward call (head dim d = 128 only).
 *
 * The pages train the video model end to end but give no gradient formulas;
 * these are the exact derivatives of the forward definition above.  With
 * L = sum(dout * out) + sum(dstate_out * state_out), per (b, h) and frame f:
 *   dnum_t = dout_t / den_t,  dden_t = -(dout_t . out_t) / den_t
 *   dq_t   = 1[q_t > 0] * ([dnum_t | dden_t] S_f^T)
 *   G_f    = sum_{t in f} phi(q_t)^T [dnum_t | dden_t] + a_{f+1} G_{f+1},
 *            G_{frames-1} adds dstate_out       (G_f = dL/dS_f, d x (d+1))
 *   dk_t   = 1[k_t > 0] * ([v_t | 1] G_f^T),   dv_t = phi(k_t) G_f[:, :d]
 *   dgate_logits[b, f, h] = a_f (1 - a_f) <G_f, S_{f-1}>,  dstate_in = a_0 G_0
 * The forward states are recomputed (nothing is saved between the calls;
 * gla_forward_train and gla_backward_saved keep them instead).
 *
 * Arguments (device pointers):
 *   q, k, v, gate_logits, state_in, B, H, frames, tokens_per_frame, eps
 *                 exactly as given to gla_forward (state_in may be NULL).
 *   dout          bf16 [B, frames * tokens_per_frame, H, d], 16-byte aligned.
 *   dstate_out    fp32 [B, H, d, d + 1] or NULL (zero).
 *   dq, dk, dv    bf16 outputs, same shape and alignment as q; must not
 *                 overlap any input.
 *   dgate_logits  fp32 [B, frames, H] output; must not be NULL when
 *                 B * H * frames > 0.
 *   dstate_in     fp32 [B, H, d, d + 1] output or NULL (not written).  Written
 *                 even when state_in is NULL (the gradient at the zero state).
 *   d             must be 128 (GLA_ERR_UNSUPPORTED_D otherwise).
 * Memory: a workspace of about (B*H*frames*10 + #SMs*4) * (d+1)*d bytes from
 * the same pool as gla_forward, freed on `stream`.  Return codes and error
 * behaviour as gla_forward.
 */
int gla_backward(const void* q, const void* k, const void* v,
                 const float* gate_logits, const float* state_in,
                 const void* dout, const float* dstate_out,
                 void* dq, void* dk, void* dv,
                 float* dgate_logits, float* dstate_in,
                 int B, int H, int frames, int tokens_per_frame, int d,
                 float eps, cudaStream_t stream);

/*
 * gla_backward_timed -- gla_backward that records seven caller-created CUDA
 * events on `stream`: events[0] before the first kernel and events[i] after
 * the i-th of the six kernels (state increments, forward scan, query-side
 * gradients, reverse scan, gate gradients, key/value gradients).  `events`
 * is a host array of 7 cudaEvent_t.
 */
int gla_backward_timed(const void* q, const void* k, const void* v,
                       const float* gate_logits, const float* state_in,
                       const void* dout, const float* dstate_out,
                       void* dq, void* dk, void* dv,
                       float* dgate_logits, float* dstate_in,
                       int B, int H, int frames, int tokens_per_frame, int d,
                       float eps, cudaStream_t stream, cudaEvent_t* events);

/*
 * gla_saved_bytes -- size in bytes of the context gla_forward_train saves for
 * gla_backward_saved: per (b, f, h) the frame's state S_f as the bf16 image
 * the output kernel reads, its bf16 remainder and S_f in fp32, i.e. about
 * B*H*frames*4*(d+1)*d bytes (133 MB for B=2, H=24, 21 frames, d=128).
 * 0 when d != 128 or a size is negative.  Host-only; no CUDA call.
 */
size_t gla_saved_bytes(int B, int H, int frames, int tokens_per_frame, int d);

/*
 * gla_forward_train -- gla_forward (head dim d = 128, plain layer) that also
 * writes the per-frame states into `saved`, so that the backward pass of the
 * same call does not recompute them (gla_backward_saved).  out and state_out
 * are the same as gla_forward's, bit for bit.
 *   saved   device buffer of gla_saved_bytes(B, H, frames, tokens_per_frame,
 *           d) bytes, 256-byte aligned, owned by the caller; its contents are
 *           opaque and valid for the backward of this call's inputs (q, k, v,
 *           gate_logits, state_in) only.  Must not be NULL when
 *           B * H * frames > 0 (GLA_ERR_NULL), nor overlap any argument.
 * Other arguments, memory and return codes as gla_forward; d != 128 gives
 * GLA_ERR_UNSUPPORTED_D.  Single-frame calls write every unit's state
 * through the scan kernel (the increment kernel's fold is not used).
 */
int gla_forward_train(const void* q, const void* k, const void* v,
                      const float* gate_logits, const float* state_in, float* state_out,
                      void* out, void* saved, int B, int H, int frames, int tokens_per_frame,
                      int d, float eps, cudaStream_t stream);

/*
 * gla_backward_saved -- gla_backward from the context `saved` that
 * gla_forward_train wrote for the same inputs: the state increments and the
 * forward scan are not run again (four kernels instead of six), and the
 * gradients are the same as gla_backward's, bit for bit.  `saved` is read
 * only.  The arguments are gla_backward's plus `saved` (NULL: GLA_ERR_NULL
 * when B * H * frames > 0; 256-byte aligned: GLA_ERR_ALIGN otherwise).  A
 * context from other inputs gives wrong gradients and is not detected.
 * Memory: a workspace of about (B*H*frames*8 + #SMs*4) * (d+1)*d bytes.
 */
int gla_backward_saved(const void* q, const void* k, const void* v,
                       const float* gate_logits, const float* state_in, const void* saved,
                       const void* dout, const float* dstate_out,
                       void* dq, void* dk, void* dv,
                       float* dgate_logits, float* dstate_in,
                       int B, int H, int frames, int tokens_per_frame, int d,
                       float eps, cudaStream_t stream);

/*
 * gla_backward_saved_timed -- gla_backward_saved that records seven
 * caller-created CUDA events on `stream` in gla_backward_timed's places (the
 * first three are back to back: no increment or forward-scan kernel runs).
 */
int gla_backward_saved_timed(const void* q, const void* k, const void* v,
                             const float* gate_logits, const float* state_in,
                             const void* saved, const void* dout, const float* dstate_out,
                             void* dq, void* dk, void* dv,
                             float* dgate_logits, float* dstate_in,
                             int B, int H, int frames, int tokens_per_frame, int d,
                             float eps, cudaStream_t stream, cudaEvent_t* events);

/*
 * gla_trim_workspace -- release the current device's unused workspace memory
 * held by the library's pool (memory of calls still in flight is kept).
 * Returns GLA_OK, GLA_ERR_DEVICE or GLA_ERR_LAUNCH.
 */
int gla_trim_workspace(void);

/*
 * gla_set_workspace_retention -- how much freed workspace memory the current
 * device's pool keeps mapped between calls (its release threshold, bytes).
 * The default keeps all of it (a later call of the same size then maps
 * nothing; measured at 720p-60s, 4.72 -> 3.79 ms per call), so after a large
 * call the pool holds up to that call's workspace (about 0.6 GB at 720p-60s)
 * until gla_trim_workspace().  A caller that runs its own caching allocator
 * beside this library can pass 0 (return everything at each synchronisation)
 * or a budget.  Creates the pool if needed.
 * Returns GLA_OK, GLA_ERR_DEVICE or GLA_ERR_LAUNCH.
 */
int gla_set_workspace_retention(unsigned long long bytes);

/*
 * Testing hooks for the failure paths (no counterpart in the paper).  They
 * make the library fail on purpose, without a GPU fault:
 *
 * gla_inject_alloc_failure -- the next `count` workspace allocations (of any
 *   entry point that allocates; not gla_forward_noalloc) fail as if the pool
 *   had no memory left: the call returns GLA_ERR_ALLOC and enqueues nothing.
 *   count = 0 disarms it.  Host only.  Returns GLA_OK.
 *
 * gla_set_wait_limit_ns -- the time after which a kernel gives up a barrier
 *   wait on the current device (default one second; ns = 0 restores it).
 *   Returns GLA_OK or GLA_ERR_LAUNCH.
 *
 * gla_inject_stall -- the next launch of the state-increment kernel on the
 *   current device withholds, on its first CTA, the loads of the tile with
 *   index `tile` in that CTA's sequence (0 = its first tile), once.  The wait
 *   for that tile runs out after the wait limit; the kernel then sets bit 0
 *   of the fault word (gla_device_fault), lets its copies in flight land,
 *   frees its tensor memory and returns, and that call's outputs are invalid.
 *   The next call runs normally.  tile < 0 disarms it.
 *   Returns GLA_OK or GLA_ERR_LAUNCH.
 */
int gla_inject_alloc_failure(int count);
int gla_set_wait_limit_ns(unsigned long long ns);
int gla_inject_stall(long long tile);

/* Static string for a gla_status code (never NULL). Host only, no CUDA call. */
const char* gla_error_string(int status);

/*
 * gla_device_fault -- synchronises `stream`, then reads and clears the
 * library's device-side fault word of the current device.  Nonzero means a
 * kernel gave up a bounded wait (about one second unless
 * gla_set_wait_limit_ns changed it) and returned early; its
 * output is then invalid.  Bit 0: state-increment kernel, bit 1: output
 * kernel, bit 2: forward scan, bit 3: reverse scan, bit 4: key/value
 * gradient kernel, bit 5: query gradient kernel, bit 6: delta-rule scan,
 * bit 7: softmax anchor kernel.
 * `code` is a host pointer.
 * Returns GLA_OK or GLA_ERR_LAUNCH.
 */
int gla_device_fault(cudaStream_t stream, unsigned int* code);

/* Library version as major * 10000 + minor * 100 + patch.  Host only. */
int gla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GLA_H_ */
