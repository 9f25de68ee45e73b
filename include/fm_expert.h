/*
 * fm_expert.h -- C ABI of the B200 (sm_100a) flow-matching action-expert
 * denoise loop.
 *
 * What the library computes (the pages print no formula; every convention
 * below is this library's reading, stated where it is used):
 *
 *   "LingBot-VLA on Thor (sm_110)", §1 Architecture / shapes: a 36-layer
 *   flow-matching action expert, action chunk [1, 50, 75], denoise step count
 *   10 / 25 / 50.  §2 Build: fused AdaRMSNorm, SwiGLU tail, QKV + RoPE.
 *   §3 FlashAttention-4: grouped-query denoise attention.  §6 Notes: all
 *   buffers pre-allocated, the loop captured in a CUDA graph, shapes fixed
 *   per graph.
 *   "LingBot-VLA v2 Examples", Configuration / CUDA Graph: the 36-layer
 *   prefix KV cache is built per request and reused by all denoise steps; a
 *   new instruction reuses the same denoise graph (here: fm_set_prefix never
 *   forces a recapture).
 *
 * One velocity evaluation v(x, t) for a chunk x [T, A] (T = chunk_len):
 *   m      = SiLU(sinusoid256(t) W1^T) W2^T, cut per layer into
 *            (s_a, b_a, g_a, s_f, b_f, g_f) and a final (s_o, b_o)
 *   h      = x W_in^T
 *   per layer l:
 *     y    = h (mean(h^2) + eps)^-1/2 (1 + s_a) + b_a
 *     q,k,v= y Wq^T, y Wk^T, y Wv^T; rotate-half RoPE on q, k at P .. P+T-1
 *     o    = softmax(q K^T / sqrt(hd)) V over [prefix K/V ; chunk k/v],
 *            query head h reading KV head h / (H_q / H_kv), no mask
 *     h   += g_a * (o Wo^T)
 *     y    = AdaRMSNorm(h; s_f, b_f)
 *     h   += g_f * ((SiLU(y Wg^T) * (y Wu^T)) Wd^T)
 *   v      = AdaRMSNorm(h; s_o, b_o) W_out^T (+ out_bias)
 * and fm_denoise integrates x <- x + dt v(x, t_k), t_k = 1 - k/n, dt = -1/n.
 *
 * Conventions of every entry point:
 *   * Matrices are row-major W[out, in]; bf16 values are passed as their
 *     16-bit patterns (uint16_t).  Activations handed in or out are fp32.
 *   * Pointers marked "host or device" are classified with
 *     cudaPointerGetAttributes; host memory may be pageable or pinned.
 *   * `stream` is a cudaStream_t (NULL = legacy default stream).  Calls on
 *     device buffers are stream-ordered and asynchronous; a call that writes
 *     to a host buffer synchronises `stream` before it returns.
 *   * A handle is not thread-safe: use it from one host thread (and one
 *     stream at a time).  Different handles are independent.
 *   * On error the call returns a non-zero fm_status, leaves outputs
 *     unspecified, and fm_last_error(handle) describes the failure.  A device
 *     wait that exceeds its bound is reported as FM_ERR_TIMEOUT by the next
 *     call that synchronises (fm_sync, or any call writing host memory).
 */
#ifndef FM_EXPERT_H
#define FM_EXPERT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FM_ABI_VERSION 1

typedef enum fm_status {
  FM_OK = 0,
  FM_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, size beyond capacity   */
  FM_ERR_NOT_READY = 2,     /* fm_set_prefix has not been called for this batch */
  FM_ERR_OOM = 3,           /* device allocation failed                         */
  FM_ERR_CUDA = 4,          /* a CUDA call failed (text in fm_last_error)       */
  FM_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up               */
  FM_ERR_UNSUPPORTED = 6    /* shape or device the library does not support     */
} fm_status;

typedef enum fm_wtype {
  FM_W_BF16 = 0,            /* per-layer linears kept in bf16                   */
  FM_W_FP8_E4M3 = 1,        /* per-layer linears quantised to E4M3, one fp32
                               scale per output row (s = absmax / 448)          */
  FM_W_FP8_NVFP4_GU = 2,    /* E4M3 as above for wq/wk/wv/wo/w_down; w_gate and
                               w_up in NVFP4: E2M1 codes, one E4M3 scale per 16
                               inputs, one fp32 scale per tensor ("LingBot-VLA
                               on Thor (sm_110)", §1: FP8 weights with an FP4
                               gate_up)                                          */
  FM_W_W8A8_E4M3 = 3        /* E4M3 weights as FM_W_FP8_E4M3 and E4M3 inputs of
                               the four per-layer linears, one fp32 scale per
                               token row (s = amax_row / 448); every batch size
                               runs on the batched tensor-core path (kind::f8f6f4
                               MMAs).  Needs d_model a multiple of 256 and at
                               most 1024, n_q_heads*head_dim and d_ff multiples
                               of 256 and at most 4096, head_dim 64 or 128.
                               The trace and profile hooks of the one-request
                               kernel return FM_ERR_UNSUPPORTED.                 */
} fm_wtype;

/* Model shape and capacities.  Requirements (checked by fm_expert_create):
 * d_model, d_ff and n_q_heads*head_dim multiples of 64; head_dim even and
 * <= 128; n_q_heads a multiple of n_kv_heads; chunk_len <= 50 rows per
 * request fit one 64-row tile; action_dim <= 128; max_steps <= 64. */
typedef struct fm_config {
  int n_layers;      /* L: transformer layers of the expert (36)              */
  int d_model;       /* d: residual width (1024)                              */
  int n_q_heads;     /* H_q (16)                                              */
  int n_kv_heads;    /* H_kv (2)                                              */
  int head_dim;      /* hd (128)                                              */
  int d_ff;          /* F: SwiGLU width (4096)                                */
  int action_dim;    /* A: action dimension (75; 55 for the v2 chunk)         */
  int chunk_len;     /* T: action horizon (50)                                */
  int max_prefix;    /* capacity for P, the prefix length                     */
  int max_batch;     /* capacity for B, requests per call                     */
  int max_steps;     /* capacity for n, Euler steps per call                  */
  float rms_eps;     /* AdaRMSNorm epsilon (1e-6)                             */
  float rope_base;   /* RoPE base (1e4)                                       */
  int wtype;         /* fm_wtype                                              */
} fm_config;

/* Per-layer weights, bf16 bits, [out, in], host or device. */
typedef struct fm_layer_weights {
  const uint16_t *wq;      /* [H_q*hd, d]   query projection                 */
  const uint16_t *wk;      /* [H_kv*hd, d]  key projection                   */
  const uint16_t *wv;      /* [H_kv*hd, d]  value projection                 */
  const uint16_t *wo;      /* [d, H_q*hd]   attention output projection      */
  const uint16_t *w_gate;  /* [F, d]        SwiGLU gate                      */
  const uint16_t *w_up;    /* [F, d]        SwiGLU up                        */
  const uint16_t *w_down;  /* [d, F]        SwiGLU down                      */
} fm_layer_weights;

typedef struct fm_weights {
  const uint16_t *time_w1;   /* [d, 256]           time MLP, first linear    */
  const uint16_t *time_w2;   /* [L*6*d + 2*d, d]   time MLP, second linear   */
  const uint16_t *in_proj;   /* [d, A]             action in-projection      */
  const uint16_t *out_proj;  /* [A, d]             action out-projection     */
  const float *out_bias;     /* [A] fp32 or NULL: constant added to v (a test
                                hook to build a constant velocity field)     */
  const fm_layer_weights *layers;   /* [L], host memory                      */
} fm_weights;

typedef struct fm_expert fm_expert;

/* Create a handle on `device`.  COPIES every weight into a library-owned,
 * kernel-ready arena (and, for FM_W_FP8_E4M3 / FM_W_FP8_NVFP4_GU /
 * FM_W_W8A8_E4M3, quantises the per-layer linears itself); the caller may free its copies when the call
 * returns.  Allocates every buffer the loop needs for the capacities in
 * `cfg`; a bf16 handle with max_batch >= 2 also packs the weights a second
 * time in the batched path's tile layout (B >= 2 requests then advance through
 * each Euler step together as M = B*T-row tensor-core GEMMs); a
 * FM_W_W8A8_E4M3 handle packs only that layout, in E4M3.
 * Returns FM_ERR_INVALID_ARG for a bad config, FM_ERR_UNSUPPORTED for a
 * device that is not sm_100 or a W8A8 shape the batched path cannot take,
 * FM_ERR_OOM when the arena does not fit. */
fm_status fm_expert_create(const fm_config *cfg, const fm_weights *w, int device,
                           fm_expert **out);

/* Load the cached prefix K/V of `batch` requests, P = prefix_len rows each:
 * k[l], v[l] point to bf16 bits [batch, P, H_kv, hd] (host or device), one
 * pointer per layer; K is taken as already rotated.  The data is copied into
 * the handle's fixed-capacity cache; P and the RoPE positions P .. P+T-1 are
 * stored on the device, so graphs captured earlier stay valid ("LingBot-VLA
 * v2 Examples", CUDA Graph: new instructions reuse the denoise graph).
 * Requires 0 <= prefix_len <= max_prefix and 1 <= batch <= max_batch. */
fm_status fm_set_prefix(fm_expert *h, const uint16_t *const *k, const uint16_t *const *v,
                        int batch, int prefix_len, void *stream);

/* As fm_set_prefix, with a prefix length per request: k[l], v[l] point to
 * bf16 bits [batch, p_pad, H_kv, hd] (host or device) in which request b
 * holds prefix_lens[b] valid rows (0 <= prefix_lens[b] <= p_pad <=
 * max_prefix; the remaining rows are padding and are never read).  Request
 * b then attends to its P_b prefix keys plus the chunk, and its chunk tokens
 * take RoPE positions P_b .. P_b+T-1.  prefix_lens is a host array of `batch`
 * ints; the lengths are stored on the device, so a graph captured for this
 * (batch, steps) serves any lengths without recapture ("LingBot-VLA v2
 * Examples", Configuration / CUDA Graph: different language padding masks
 * reuse the same denoising graph; "api.py", state_prompt_mode "fixed": one
 * graph at the padded length masked by a device-side valid length).
 * FM_ERR_INVALID_ARG for a length outside [0, p_pad] or p_pad > max_prefix. */
fm_status fm_set_prefix_varlen(fm_expert *h, const uint16_t *const *k, const uint16_t *const *v,
                               int batch, const int *prefix_lens, int p_pad, void *stream);

/* Per-layer prefix K/V projection weights of the vision-language backbone
 * that fills the cache the expert attends to: bf16 bits [H_kv*hd, d_prefix]
 * each, [out, in], host or device. */
typedef struct fm_prefix_weights {
  const uint16_t *wk;
  const uint16_t *wv;
} fm_prefix_weights;

/* Load the prefix cache builder: w[l] for every layer l (copied and packed;
 * the caller may free them on return).  d_prefix: the backbone's hidden
 * width, a positive multiple of 64.  Call once per handle; allocates the
 * builder's device buffers (sized for max_batch x max_prefix rows).
 * FM_ERR_UNSUPPORTED when 2 * H_kv * hd is not a multiple of 128. */
fm_status fm_set_prefix_builder(fm_expert *h, const fm_prefix_weights *w, int d_prefix);

/* Build the prefix cache on the device from each layer's prefix hidden
 * states ("LingBot-VLA v2 Examples", Configuration / CUDA Graph: the 36-layer
 * KV-cache construction runs once per request, before the fixed-shape
 * denoising steps): for layer l and request b,
 *   K = RoPE(x Wk^T) at positions 0 .. P-1,  V = x Wv^T   (bf16 in the cache)
 * with x = hidden[l][b] ([prefix_len, d_prefix] bf16 bits; hidden[l] is
 * [batch, prefix_len, d_prefix], host or device).  It replaces fm_set_prefix
 * for this batch (every request gets P = prefix_len) and runs as tensor-core
 * GEMMs with a RoPE epilogue writing straight into the cache.
 * Synchronises `stream`.  FM_ERR_NOT_READY without fm_set_prefix_builder. */
fm_status fm_build_prefix(fm_expert *h, const uint16_t *const *hidden, int batch, int prefix_len,
                          void *stream);

/* Test hook: the cached prefix rows of `request` at `layer`, bf16 bits
 * [P_b, H_kv, hd] into host buffers k and v (K as stored, i.e. rotated). */
fm_status fm_get_prefix_kv(fm_expert *h, int layer, int request, uint16_t *k, uint16_t *v);

/* Denoise `batch` chunks: x0 and out are fp32 [batch, T, A], host or device
 * (independently); out may alias x0.  Runs the time MLP once, then `steps`
 * Euler steps from t = 1 to t = 0 ("LingBot-VLA on Thor (sm_110)", §1: the
 * denoise step count is configurable, 10 / 25 / 50).  The first call for a
 * given (batch, steps) captures a CUDA graph; later calls replay it.
 * batch must equal the batch of the last fm_set_prefix (else
 * FM_ERR_NOT_READY); 1 <= steps <= max_steps. */
fm_status fm_denoise(fm_expert *h, const float *x0, int batch, int steps, float *out,
                     void *stream);

/* Test hook: one velocity evaluation v(x, t_k) with t_k = 1 - step_index/steps,
 * without the Euler update.  x, v_out: fp32 [batch, T, A], host or device. */
fm_status fm_velocity(fm_expert *h, const float *x, int batch, int step_index, int steps,
                      float *v_out, void *stream);

/* Test hook: the modulation rows m_k for t_k = 1 - k/steps, k < steps, as
 * fp32 [steps, L*6*d + 2*d] into m_out (host or device). */
fm_status fm_time_modulation(fm_expert *h, int steps, float *m_out, void *stream);

/* Test hook: per-layer intermediates of one velocity evaluation for request 0
 * (batch must be 1).  Writes, into host memory `trace` of fm_trace_bytes()
 * bytes, for each layer l in order (T = chunk_len):
 *   h_in  fp32 [T, d]           residual stream entering the layer
 *   q     fp32 [T, H_q*hd]      query after RoPE (bf16 values, widened)
 *   k     fp32 [T, H_kv*hd]     chunk key after RoPE (bf16 values)
 *   v     fp32 [T, H_kv*hd]     chunk value (bf16 values)
 *   o     fp32 [T, H_q*hd]      attention output (bf16 values)
 *   h_mid fp32 [T, d]           after the attention residual
 *   u     fp32 [T, F]           SwiGLU product (bf16 values)
 *   h_out fp32 [T, d]           after the FFN residual
 * then v fp32 [T, A].  Synchronises `stream`. */
size_t fm_trace_bytes(const fm_expert *h);
fm_status fm_trace_velocity(fm_expert *h, const float *x, int step_index, int steps,
                            float *trace, void *stream);

/* Test hook: the E4M3 codes [out, in] and fp32 row scales [out] the handle
 * holds for per-layer linear `which` (0 wq, 1 wk, 2 wv, 3 wo, 4 w_gate,
 * 5 w_up, 6 w_down) of `layer`; host buffers, read back from the arena the
 * kernels stream (for FM_W_W8A8_E4M3 the batched GEMM's tile arena).
 * FM_ERR_INVALID_ARG for a bf16 handle. */
fm_status fm_get_fp8_weights(fm_expert *h, int layer, int which, uint8_t *codes,
                             float *scale);

/* Test hook: the NVFP4 weights of w_gate (which = 4) or w_up (5) of `layer`
 * in a FM_W_FP8_NVFP4_GU handle, read back from the packed arena: codes
 * [out, in] one E2M1 code (0..15, bit 3 = sign) per byte, block scales
 * [out, in/16] E4M3 codes, and the tensor's fp32 scale g; host buffers.
 * Dequantised weight = e2m1(code) * e4m3(block scale) * g. */
fm_status fm_get_nvfp4_weights(fm_expert *h, int layer, int which, uint8_t *codes,
                               uint8_t *block_scales, float *g);

/* Test hook: R11 per-token E4M3 of `M` bf16 rows x[M, K] (host or device)
 * with the row-quantiser kernel of the W8A8 path (the pass that follows
 * attention and SwiGLU): s_m = amax_m / 448 and r_m = 448 / amax_m in fp32
 * (both 1 for a zero row), codes = E4M3(x r_m) with the product in fp32,
 * nearest-even, saturating.  Writes host codes
 * [M, K] and host scales [M].  K a multiple of 256 and at most 4096.
 * Allocates and frees temporary device memory; synchronises `stream`. */
fm_status fm_quantize_act_e4m3(fm_expert *h, const uint16_t *x, int M, int K, uint8_t *codes,
                               float *scales, void *stream);

/* Profiling hook: runs `iters` times the two kernels of one denoise (the
 * time MLP, then the denoise loop for every request) outside any graph, with
 * CUDA events on `stream` around each, and writes their mean durations in
 * milliseconds to ms[0] (time MLP) and ms[1] (loop).  Advances the handle's
 * internal chunk state; synchronises `stream`. */
fm_status fm_profile_denoise(fm_expert *h, int batch, int steps, int iters, float *ms,
                             void *stream);

/* Profiling hook: one denoise of request 0 (`steps` Euler steps, outside any
 * graph) that records %globaltimer (ns) on every CTA.  With out == NULL,
 * writes the required number of uint64 values to *n and returns.  Otherwise
 * fills host `out` [n_ctas][stride], stride = 16*n_phases + 2*n_gemms +
 * 2*n_chunks: per grid-barrier-separated phase 16 marks (start, MMAs or
 * attention done, partials pushed, partials received, epilogue done,
 * barrier arrival issued, partials staged, staging synchronised, then
 * phase-specific points); per linear the MMA warp's marks
 * (activations landed, last weight chunk landed); per weight chunk the time
 * it landed, then per weight chunk the time the producer issued it.  Unused
 * slots are 0.  n_phases = steps*(2 + 5L), n_gemms = steps*4L, n_chunks =
 * steps*L*(chunks per CTA per layer, at most 32). */
fm_status fm_profile_phases(fm_expert *h, int steps, uint64_t *out, size_t *n, void *stream);

/* Test hook (per-kernel parity of the batched path, "LingBot-VLA v2
 * Examples": intermediate-tensor parity): one velocity evaluation of `batch`
 * requests (as fm_velocity) on the batched path, stopping after each kernel
 * to copy its output to the host buffer `trace` of fm_trace_batched_bytes
 * bytes: per layer, rows m = b T + t (M = batch T rows), fp32
 *   h_in [M][d], y_a [M][d], q [M][Hq hd], k [M][Hkv hd], v [M][Hkv hd],
 *   o [M][Hq hd], h_mid [M][d], y_f [M][d], u [M][F], h_out [M][d]
 * then the velocity [M][A].  y_a and y_f are the normalised GEMM inputs as the
 * GEMMs read them (on a W8A8 handle: codes x row scale); q, k are after RoPE;
 * o and u are the bf16 outputs of attention and SwiGLU.  FM_ERR_UNSUPPORTED
 * when `batch` runs on the one-request kernel.  Synchronises (slow). */
size_t fm_trace_batched_bytes(const fm_expert *h, int batch);
fm_status fm_trace_batched(fm_expert *h, const float *x, int batch, int step_index, int steps,
                           float *trace, void *stream);

/* Wait for `stream`, then report (and clear) any device-side timeout. */
fm_status fm_sync(fm_expert *h, void *stream);

/* Test hook for failure detection (the pages' release checks cover fault and
 * shutdown handling; this is the device-side half).  While `on` is non-zero,
 * the one-request loop kernel of this handle expects one writer more than
 * exists at its QKV -> attention hand-off, so that wait can never complete,
 * and every wait of the loop kernel gives up after `spin_cycles` SM clock
 * cycles (0: the default of about 2 s).  The launch then ends early with the
 * handle's error word set, and the next synchronising call returns
 * FM_ERR_TIMEOUT; the device context stays usable.  Off by default.  Blocks
 * until the device is idle and drops the handle's captured graphs, so later
 * calls see the setting.  FM_ERR_INVALID_ARG for a negative spin_cycles. */
fm_status fm_test_stall(fm_expert *h, int on, long long spin_cycles);

/* Launch geometry the handle chose: CTAs per cluster, clusters, CTAs. */
fm_status fm_get_geometry(const fm_expert *h, int *cluster_size, int *n_clusters,
                          int *n_ctas);

/* The time-conditioning rows m_k (as fm_time_modulation) for callers that
 * cannot allocate device memory: a control loop or runtime whose device memory
 * is fixed and audited at start-up, or an embedder that gives the library
 * only buffers it owns.  The pages have no counterpart of this entry point;
 * it allocates nothing.
 *   w1: device bf16 bits [d_model, 256]; w2: device bf16 bits [n_mod, d_model]
 *   (row-major, as in fm_weights); m_out: device fp32 [steps, n_mod].  All three
 *   must be 4-byte aligned.
 *   Limits: 1 <= steps <= 64, 64 <= d_model <= 1024 (a multiple of 64).  Larger
 *   sizes and misaligned pointers return FM_ERR_INVALID_ARG and
 *   fm_last_error(NULL) says why.
 * Its only intermediate, the bf16 hidden activations (64 x 1024 at most, 128
 * KB), lives in a device array inside the library that every GPU using the
 * library holds until the process exits.  The first call on a device (and the
 * first after cudaDeviceReset on it) looks up that array's address; make that
 * first call before any stream capture.  Its kernels use no local-memory
 * stack.  All
 * calls share the array and each overwrites the part it reads, so nothing
 * depends on a previous call; calls that overlap on the GPU (two streams)
 * race on it.  Stream-ordered; does not synchronise. */
fm_status fm_time_modulation_noalloc(const uint16_t *w1, const uint16_t *w2, int d_model, int n_mod,
                                     int steps, float *m_out, void *stream);

/* Release the handle and every device buffer it owns; NULL is a no-op.
 * Returns the number of device bytes released. */
size_t fm_expert_destroy(fm_expert *h);

/* Text of the last error on this handle ("" if none); NULL handle: the last
 * error of a failed fm_expert_create or fm_time_modulation_noalloc on this
 * thread. */
const char *fm_last_error(const fm_expert *h);
const char *fm_status_string(fm_status s);
int fm_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FM_EXPERT_H */
