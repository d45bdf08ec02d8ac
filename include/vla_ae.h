/*
 * vla_ae.h -- C ABI of the B200 (sm_100a) flow-matching action-expert denoise loop.
 *
 * The operation: the action expert of a vision-language-action model integrates
 *     x_{k+1} = x_k + dt * v_theta(x_k, t_k, prefix KV),   t_k = 1 - k/N,  dt = -1/N,
 * from Gaussian noise x_0 over N fixed Euler steps ("AI Infra如何优化VLA" (RimBot), section
 * 整体方案: a 4-step x 36-layer DiT action head denoising from random noise; APXInf article,
 * section "CUDA Graph、FP8 和 Rust": 10 flow steps, a 1-step variant and FP8 weights).
 * v_theta is a DiT: per layer RMSNorm + adaLN time modulation, fused QKV projection with
 * half-split RoPE, GQA attention of the action tokens over themselves and the cached VLM prefix
 * K/V, o-projection, SwiGLU MLP and gated residual adds; an action out-projection closes it.
 * ("跨XPU平台表征视觉-语言-动作模型" section 4.2: this stage is memory-bound.)
 *
 * Conventions for every entry point:
 *   - returns VLA_AE_OK (0) or a negative VLA_AE_E* code; no exception crosses the ABI;
 *   - calls taking a `stream` (a cudaStream_t, NULL = legacy default stream) only enqueue work
 *     and return; results are ready when that stream reaches the enqueued work;
 *   - a handle is not thread-safe; different handles are independent;
 *   - the library allocates and owns all of its device memory; caller pointers are borrowed for
 *     the duration of the call (or, for asynchronous calls, until the stream has consumed them).
 * Data types: "bf16" = IEEE bfloat16 bit patterns (uint16), "fp32" = IEEE float.
 */
#ifndef VLA_AE_H
#define VLA_AE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status codes */
#define VLA_AE_OK 0
#define VLA_AE_EINVAL (-1)       /* bad argument: null pointer, dims out of range, n_prefix > max */
#define VLA_AE_ENOMEM (-2)       /* device allocation failed */
#define VLA_AE_ECUDA (-3)        /* a CUDA runtime call failed (no device, launch error, ...) */
#define VLA_AE_ENOPREFIX (-4)    /* vla_ae_denoise before any vla_ae_set_prefix */
#define VLA_AE_ETIMEOUT (-5)     /* a bounded device-side wait ran out (see vla_ae_status) */
#define VLA_AE_EUNSUPPORTED (-6) /* valid dims the library does not implement (e.g. head_dim) */

/* ------------------------------------------------------------------ configuration */
/* Weight formats of the per-layer linears.  FP8_E4M3: the FP8 weights of the APXInf article
 * (section "CUDA Graph、FP8 和 Rust").  INT8: the INT8 quantisation the same section names for
 * GPUs without FP8 tensor cores (Jetson Orin), here weight-only with one scale per output channel.
 * INT4_G128: INT4, named next to FP8 in "AI Infra如何优化VLA" (section 后续工作), here W4A16 with
 * one scale per output channel and group of 128 inputs. */
typedef enum { VLA_AE_BF16 = 0, VLA_AE_FP8_E4M3 = 1, VLA_AE_INT8 = 2, VLA_AE_INT4_G128 = 3 } vla_ae_wtype;

/* Model and workload dimensions, fixed at create time.
 * Requirements (else VLA_AE_EINVAL): every count >= 1 except has_state_token (0/1) and
 * max_prefix (>= 0); hidden, inter % 8 == 0; head_dim in {64, 128, 256};
 * n_q_heads % n_kv_heads == 0; t_emb_dim even; action_dim <= 64;
 * batch * (n_action_tokens + has_state_token) <= 4096. */
typedef struct {
  int n_layers;         /* DiT layers L */
  int hidden;           /* H */
  int n_q_heads;        /* nq */
  int n_kv_heads;       /* nkv (GQA: consecutive q heads share a kv head) */
  int head_dim;         /* hd; q width nq*hd may differ from H */
  int inter;            /* SwiGLU intermediate I */
  int t_emb_dim;        /* sinusoidal time-embedding width Dt */
  int action_dim;       /* A */
  int n_action_tokens;  /* T (action chunk length) */
  int has_state_token;  /* 1: one proprioceptive state token precedes the action tokens */
  int max_prefix;       /* largest prefix length P accepted by vla_ae_set_prefix */
  int batch;            /* B independent samples per call */
  float rope_theta;     /* RoPE base (10000) */
  float rms_eps;        /* RMSNorm epsilon (1e-6) */
  int wtype;            /* vla_ae_wtype of the per-layer q/k/v/o/gate/up/down weights */
} vla_ae_dims;

/* Weights: bf16, matrices [out][in] row-major.  Per-layer entries are arrays of n_layers
 * pointers.  adaLN per layer: w_ada [6H][Dt], b_ada [6H] in the order shift/scale/gate for the
 * attention branch then for the MLP branch; final adaLN w_fada [2H][Dt], b_fada [2H] (shift,
 * scale).  wq [nq*hd][H], wk/wv [nkv*hd][H], wo [H][nq*hd], wg/wu [I][H], wd [H][I];
 * w_in/w_state [H][A], b_in/b_state [H], w_out [A][H], b_out [A]; w_state/b_state are ignored
 * (may be NULL) without a state token.  on_device: 1 = all pointers are device memory,
 * 0 = host memory; device per-layer matrices must be 16-byte aligned.  With wtype FP8 the
 * library quantises q/k/v/o/gate/up/down itself (one fp32 scale per output channel, scale =
 * max|w|/448, codes = e4m3 round-to-nearest-even saturating of w/scale); with wtype INT8 likewise
 * with scale = max|w|/127 and codes = round-to-nearest-even of w/scale clamped to [-127, 127]
 * (a zero row takes scale 1); with wtype INT4_G128 per output channel and group of 128 inputs
 * with scale = max|w_group|/7 and codes clamped to [-7, 7], the tensor cores then multiply
 * bf16(code * scale); everything else stays bf16.  The caller keeps ownership; the library
 * copies. */
typedef struct {
  const void *w_in, *b_in, *w_state, *b_state;
  const void *const *w_ada, *const *b_ada;
  const void *const *wq, *const *wk, *const *wv, *const *wo;
  const void *const *wg, *const *wu, *const *wd;
  const void *w_fada, *b_fada, *w_out, *b_out;
  int on_device;
} vla_ae_weights;

typedef struct vla_ae *vla_ae_t;

/* Create a handle on the current CUDA device: validates dims, allocates every device buffer the
 * loop needs, packs (and for FP8 quantises) the weights into the kernels' streaming layout.
 * Synchronous.  Errors: EINVAL, EUNSUPPORTED, ENOMEM, ECUDA; *out is NULL on error. */
int vla_ae_create(const vla_ae_dims *dims, const vla_ae_weights *weights, vla_ae_t *out);

/* Set the cached VLM prefix for the next denoise calls (once per control cycle).
 *   k, v   bf16 [B][L][n_prefix][nkv][hd], keys already rotated (RoPE applied by the VLM);
 *   state  bf16 [B][A] proprioceptive state (required iff has_state_token, else ignored);
 *   on_device: 1 = device pointers (copied device-to-device), 0 = host pointers.
 * 0 <= n_prefix <= max_prefix.  Self tokens take positions n_prefix .. n_prefix+Ts-1.
 * Asynchronous on `stream`.  Errors: EINVAL, ECUDA. */
int vla_ae_set_prefix(vla_ae_t h, const void *k, const void *v, int n_prefix, const void *state,
                      int on_device, void *stream);

/* Allocation-free variant of vla_ae_set_prefix for host buffers.  The pages have no counterpart:
 * it exists for callers that cannot allocate device memory while they run, such as a robot control
 * loop that must not pay the allocator's unbounded latency every cycle, or code running while a
 * CUDA graph is being captured on the device (an allocation there is not allowed).  Where
 * vla_ae_set_prefix with host pointers stages the prefix through buffers it allocates, this call
 * stages it one layer at a time through a fixed device array of VLA_AE_STATIC_SCRATCH_BYTES
 * (16 MiB) compiled into the library; every GPU that loads the library holds that array until
 * the process exits.  It allocates nothing and frees nothing.
 *   k, v   host bf16 [B][L][n_prefix][nkv][hd] (pinned memory gives asynchronous copies);
 *   state  host bf16 [B][A] (required iff has_state_token).
 * One layer of K and V for the whole batch, batch * n_prefix * nkv * hd * 4 bytes, must fit in
 * the array, else VLA_AE_EINVAL (with a message on stderr).  All calls share the one array, which
 * keeps the last call's contents (nothing in it needs to start at zero): calls that overlap on
 * the GPU (other streams, other handles on the same device) race on it, so serialise them.  The
 * first call on a device looks up the array's device address (cudaGetSymbolAddress); make that
 * first call before any stream capture.  Asynchronous on `stream`.  Errors: EINVAL, ECUDA. */
#define VLA_AE_STATIC_SCRATCH_BYTES (16u << 20)
int vla_ae_set_prefix_static(vla_ae_t h, const void *k, const void *v, int n_prefix, const void *state,
                             void *stream);

/* Run the N-step Euler loop.
 *   noise  device bf16 [B][T][A], the initial x_0;
 *   steps  N >= 1 (t_k = 1 - k/N, dt = -1/N);
 *   out    device fp32 [B][T][A], receives x_N (caller-owned).
 * The first call for a given `steps` builds that step count's adaLN table and captures the
 * loop as one CUDA graph (do it before timing); later calls replay it.  Asynchronous on
 * `stream`.  Errors: EINVAL, ENOPREFIX, ECUDA. */
int vla_ae_denoise(vla_ae_t h, const void *noise, int steps, float *out, void *stream);

/* ------------------------------------------------------------------ prefix K/V producer
 * The VLM side of the cached prefix ("AI Infra如何优化VLA", section 算子开发: the backbone's pre-norm
 * RMSNorm and the half-split RoPE of the prefill): for every layer l the hidden states h_l of the
 * P prefix tokens become x = RMSNorm(h_l) * gain_l, K_l = RoPE(x Wk_l^T) at positions 0..P-1 and
 * V_l = x Wv_l^T, written straight into the loop's caches (the expert attends to the backbone's
 * K/V, so its kv heads are the backbone's).  bf16 weights; the GEMM is the QKV kernel without q
 * heads, the RMSNorm scale applied by linearity.
 *
 * vla_ae_attach_vlm_kv: copy and pack the backbone's per-layer K/V projections.
 *   hidden_vlm  Hv, the backbone's width (% 8 == 0);   rms_eps  its RMSNorm epsilon;
 *   wk, wv      [L] arrays of bf16 [nkv*hd][Hv];  gain  [L] arrays of bf16 [Hv];
 *   on_device   1: device pointers (16-byte aligned), 0: host.
 * Synchronous.  Errors: EINVAL, ENOMEM, ECUDA, EUNSUPPORTED.
 *
 * vla_ae_set_prefix_hidden: the current prefix from device bf16 hidden states [B][L][P][Hv]
 * (n_prefix <= max_prefix) and the state token as in vla_ae_set_prefix.  Asynchronous on
 * `stream`.  Errors: EINVAL (also before vla_ae_attach_vlm_kv), ECUDA. */
typedef struct {
  int hidden_vlm;
  float rms_eps;
  int on_device;
  const void *const *wk, *const *wv, *const *gain;
} vla_ae_vlm_kv_weights;
int vla_ae_attach_vlm_kv(vla_ae_t h, const vla_ae_vlm_kv_weights *w);
int vla_ae_set_prefix_hidden(vla_ae_t h, const void *hidden, int n_prefix, const void *state, void *stream);

/* Test hook: the current prefix's cached rows of layer `layer` as device fp32 k, v [B][P][nkv][hd]
 * (K after RoPE).  Synchronous.  Errors: EINVAL, ENOPREFIX, ECUDA. */
int vla_ae_debug_prefix_kv(vla_ae_t h, int layer, float *k, float *v);

/* ------------------------------------------------------------------ stale-prefix overlap
 * V-AEFusion ("跨XPU平台表征视觉-语言-动作模型" section 5.3): the first denoising steps of a control
 * cycle run on the previous cycle's prefix while the VLM computes the new one on another stream;
 * the remaining steps use the new prefix.
 *
 * vla_ae_set_prefix_next: lay out the NEXT cycle's prefix (arguments as vla_ae_set_prefix) into a
 * second set of caches, asynchronously on `stream` (typically the stream that produced it), and
 * record a library-owned event there.  The first call allocates that second set.
 *
 * vla_ae_denoise_stale: run steps [0, n_stale) of the `steps`-step loop on the current prefix,
 * make `stream` wait for the event of the last vla_ae_set_prefix_next, run steps [n_stale, steps)
 * on the next prefix (its state token included), then make the next prefix the current one.
 * 0 <= n_stale <= steps (0: all steps on the new prefix; steps: all on the old one).  Enqueue
 * vla_ae_set_prefix_next before this call (both are asynchronous: the overlap happens on the
 * GPU).  The first call per (steps, n_stale) captures two graphs.
 * Errors: EINVAL, ENOPREFIX (no current prefix, or no vla_ae_set_prefix_next since the last
 * vla_ae_denoise_stale), ECUDA. */
int vla_ae_set_prefix_next(vla_ae_t h, const void *k, const void *v, int n_prefix, const void *state, int on_device,
                           void *stream);
int vla_ae_denoise_stale(vla_ae_t h, const void *noise, int steps, int n_stale, float *out, void *stream);

/* The Euler loop along a caller-chosen time grid: n steps x_{k+1} = x_k + (t_{k+1} - t_k) *
 * v(x_k, t_k) for the host array t_grid[0..n] (strictly decreasing, finite; 1 <= n <=
 * VLA_AE_MAX_GRID_STEPS).  It serves step skipping ("跨XPU平台表征视觉-语言-动作模型" sections 5.2
 * and 5.3.2: DP-Cache drops a fixed set of intermediate diffusion steps; for Euler a dropped
 * step's interval joining the step before it equals reusing that step's velocity) and the
 * one-step variant (APXInf article, section "CUDA Graph、FP8 和 Rust"): {1, 0}.
 *   noise  device bf16 [B][T][A];  out  device fp32 [B][T][A] (caller-owned).
 * The first call for a given grid builds its tables and captures its graph (as vla_ae_denoise
 * does per step count; the uniform grid with values exactly 1 - k/n shares that step count's
 * tables).  Asynchronous on `stream`.  Errors: EINVAL (bad grid or pointers), ENOPREFIX, ECUDA. */
#define VLA_AE_MAX_GRID_STEPS 256
int vla_ae_denoise_sched(vla_ae_t h, const void *noise, const float *t_grid, int n, float *out, void *stream);

/* Same as vla_ae_denoise with host buffers: noise_host bf16 [B][T][A] and out_host fp32
 * [B][T][A] (pinned memory gives asynchronous copies).  Enqueues the host-to-device copy, the
 * loop and the device-to-host copy on `stream`; out_host is valid after the stream syncs. */
int vla_ae_denoise_host(vla_ae_t h, const void *noise_host, int steps, float *out_host, void *stream);

/* Sticky device-side status: VLA_AE_OK, or VLA_AE_ETIMEOUT when a bounded wait inside a kernel
 * ran out (the results of that call are invalid).  Synchronises the device.  Clears the flag. */
int vla_ae_status(vla_ae_t h);

/* Static text for a status code. */
const char *vla_ae_strerror(int code);

/* Release every resource of the handle (synchronises the device).  NULL is a no-op. */
void vla_ae_destroy(vla_ae_t h);

/* ------------------------------------------------------------------ introspection */
#define VLA_AE_Q_KERNELS_PER_LOOP 1   /* kernel launches per denoise loop of `arg` steps */
#define VLA_AE_Q_WEIGHT_BYTES 2       /* bytes of streamed linear weights (+fp8 scales) per step */
#define VLA_AE_Q_KV_BYTES 3           /* bytes of prefix K+V read per step (whole batch) */
#define VLA_AE_Q_DEVICE_BYTES 4       /* device memory held by the handle */
#define VLA_AE_Q_SPLITS 5             /* packed split-K of the four GEMMs: qkv | o<<8 | gu<<16 | d<<24 */
#define VLA_AE_Q_OP_BYTES 6           /* algorithmic bytes one launch of loop kernel `arg` reads from HBM:
                                         the weight matrix (+ fp8 scales) of op 0 qkv, 2 o, 3 gate/up,
                                         4 down; the layer's prefix K+V for op 1 (attention) */
#define VLA_AE_Q_ENGINE 7             /* layer engine in use: VLA_AE_ENGINE_PER_OP or VLA_AE_ENGINE_PERSISTENT */
/* Query a property of the handle into *value.  Errors: EINVAL. */
int vla_ae_query(vla_ae_t h, int what, int arg, long long *value);

/* Benchmark hook: enqueue `count` launches of one kernel of the loop (op: 0 QKV GEMM, 1 attention,
 * 2 o-projection, 3 gate/up GEMM, 4 down GEMM) for layers 0, 1, 2, ... (cycling), chained by
 * programmatic dependent launch exactly as inside the loop, with step 0 of the `steps` tables and
 * the handle's current buffers (the values computed are not meaningful).  Lets a caller time one
 * kernel with CUDA events on `stream`; weights of successive layers are distinct, so they stream
 * from HBM.  Asynchronous.  Errors: EINVAL, ENOPREFIX, ECUDA. */
int vla_ae_bench_op(vla_ae_t h, int op, int count, int steps, void *stream);

/* ------------------------------------------------------------------ layer engines
 * How the L layers of one Euler step run (the arithmetic and its order are the same):
 *   VLA_AE_ENGINE_PER_OP (0): five kernels per layer (QKV GEMM, attention, o-proj GEMM, gate/up
 *     GEMM, down GEMM) chained by programmatic dependent launch;
 *   VLA_AE_ENGINE_PERSISTENT (1): one kernel per step with one CTA per SM resident for all
 *     layers; weights stream continuously and phases hand over through device-scope counters.
 *     Available for bf16 weights with at most 128 token rows (batch x self tokens), a hidden
 *     size that is a multiple of 4, and work units that fit the SMs.
 *   VLA_AE_ENGINE_AUTO (2): the first vla_ae_denoise / _host / _sched call of a step count (or
 *     time grid) and prefix length captures the loop with both engines, times three replays of
 *     each on the caller's stream (a one-off cost of a few loops, synchronising the host once) and
 *     keeps the faster; later calls replay it.  vla_ae_denoise_stale follows the choice made for
 *     whole loops (per-op until one was made).  Without the persistent engine, AUTO is per-op.
 * create selects VLA_AE_ENGINE_PER_OP.
 * Select the engine for later denoise / debug calls (a graph captured for the other engine is
 * re-captured); VLA_AE_Q_ENGINE reports the engine in use (AUTO: the one it picked).
 * Errors: EINVAL, EUNSUPPORTED (persistent engine not available here). */
#define VLA_AE_ENGINE_PER_OP 0
#define VLA_AE_ENGINE_PERSISTENT 1
#define VLA_AE_ENGINE_AUTO 2
int vla_ae_set_engine(vla_ae_t h, int engine);

/* ------------------------------------------------------------------ test hooks
 * Teacher-forced execution of one DiT layer (per-layer parity): h_in and h_out are device fp32
 * [B*Ts][H] (row b*Ts + j is token j of sample b; j = 0 is the state token when present);
 * the layer uses the adaLN table of step `step` out of `steps` and the current prefix.
 * Any non-NULL trace pointer (device fp32) receives an intermediate, row per token:
 *   q [B*Ts][nq*hd] and k, v [B*Ts][nkv*hd] after RoPE (v unrotated), o [B*Ts][nq*hd] attention
 *   output, h_attn [B*Ts][H] after the attention residual, m [B*Ts][I] SwiGLU output.
 * Synchronous.  Errors: EINVAL, ENOPREFIX, ECUDA. */
typedef struct {
  float *q, *k, *v, *o, *h_attn, *m;
} vla_ae_trace;
int vla_ae_debug_layer(vla_ae_t h, int layer, int step, int steps, const float *h_in, float *h_out,
                       const vla_ae_trace *trace);

/* Failure-detection probe: run a kernel whose wait on an mbarrier (that nothing arrives on) is
 * bounded to `attempts` tries (1 .. 2^20).  The wait runs out, the kernel records a timeout in the
 * handle's device status word and returns; vla_ae_status then reports VLA_AE_ETIMEOUT and the
 * handle stays usable.  Synchronous.  Errors: EINVAL, ECUDA. */
int vla_ae_debug_wait_probe(vla_ae_t h, unsigned attempts);

/* v_theta(x, t_step) for device fp32 x [B][T][A] into device fp32 v [B][T][A].  Synchronous. */
int vla_ae_debug_velocity(vla_ae_t h, int step, int steps, const float *x, float *v);

/* Read back one packed per-layer weight in [out][in] order (which: 0 q, 1 k, 2 v, 3 o, 4 gate,
 * 5 up, 6 down) into host memory: bf16 weights as uint16 bits, FP8 / INT8 / INT4 weights as
 * one code per byte (e4m3 bits / two's-complement int8 / int4 sign-extended to int8) plus fp32
 * scales [out] ([out][ceil(in/128)] for INT4; scales may be NULL for bf16).  Synchronous. */
int vla_ae_debug_weight(vla_ae_t h, int layer, int which, void *w_host, float *scales_host);

#ifdef __cplusplus
}
#endif
#endif /* VLA_AE_H */
