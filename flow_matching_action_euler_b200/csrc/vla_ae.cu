// Host engine behind the C ABI in include/vla_ae.h.
//
// create:      plan every kernel of the loop (tiles, split-K cluster sizes, shared memory), allocate
//              all device buffers once ("AI Infra如何优化VLA" section CUDA Graph: preallocate the
//              buffers the captured graph uses), pack / quantise the weights.
// set_prefix:  lay the VLM prefix K / V out for the attention kernel, project the state token,
//              rebuild the RoPE table for the self-token positions.
// denoise:     first call per step count builds the adaLN table and captures the whole N-step loop
//              (1 + N * (5 L + 1) kernels chained by programmatic dependent launch) as one CUDA
//              graph (same page and section: warm-up, capture, replay; APXInf article: capture once,
//              replay every control cycle); later calls copy the noise in, replay, copy x out.
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <vector>

#include "../../include/vla_ae.h"
#include "ptx.cuh"
#include "gemm.cuh"
#include "attention.cuh"
#include "loop.cuh"
#include "misc.cuh"

using namespace vla;

namespace {

constexpr int kMaxDynSmem = 232448;      // 227 KB per CTA on sm_100
// Shared memory a streaming-GEMM CTA may plan for: one CTA per SM with a deep weight ring.  Two
// CTAs of ~110 KB (a dependent kernel's CTAs prefetching beside the running one) measured 5 %
// (StarVLA) to 13 % (pi0.5) slower per loop than the deeper rings.
constexpr int kGemmSmemBudget = 220 * 1024;

#define CK(call)                                                            \
  do {                                                                      \
    cudaError_t e_ = (call);                                                \
    if (e_ != cudaSuccess) {                                                \
      std::fprintf(stderr, "vla_ae: %s failed: %s (%s:%d)\n", #call,        \
                   cudaGetErrorString(e_), __FILE__, __LINE__);             \
      return e_ == cudaErrorMemoryAllocation ? VLA_AE_ENOMEM : VLA_AE_ECUDA; \
    }                                                                       \
  } while (0)

int ceil_div(int a, int b) { return (a + b - 1) / b; }
size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

enum OpId { OP_QKV = 0, OP_O = 1, OP_GU = 2, OP_D = 3 };

struct OpPlan {
  int O = 0, K = 0, Mt = 0, KB = 0, KBt = 0, S = 1, stages = 1, mpc = 1;
  size_t wbytes = 0;        // packed tile bytes of one layer
  size_t woff = 0;          // offset inside a layer's packed block
  size_t soff = 0;          // offset of the op's scales inside a layer's scale block (floats)
  int off_b = 0, off_conv = 0, off_bar = 0, off_misc = 0, off_vec = 0, smem = 0;
};

struct StepTables {
  int steps = 0;
  float* mod = nullptr;    // [steps][L][6H]
  float* fmod = nullptr;   // [steps][2H]
  float* cq = nullptr;     // [steps][L][Mt_qkv * 128]: W_qkv . shift_attn
  float* cg = nullptr;     // [steps][L][Mt_gu * 128]:  W_gu . shift_mlp
  unsigned* ctr = nullptr;  // persistent engine: per-step counter blocks [steps][ctr_step]
  std::vector<double> t;    // time grid t_0 > ... > t_steps
  std::vector<float> dt;    // Euler step k: t_{k+1} - t_k
  // captured graphs, one per (first step, end step, prefix slot, prefix length, engine)
  std::map<std::array<int, 5>, cudaGraphExec_t> graphs;
  // VLA_AE_ENGINE_AUTO: the engine that ran the whole loop faster, per prefix length
  std::map<int, bool> auto_loop;
};

// One prefix buffer set: the layer caches (prefix rows + the self rows the loop writes), the
// RoPE table of the self-token positions and the projected state token.
struct PrefixSlot {
  __nv_bfloat16 *kc = nullptr, *vct = nullptr;
  float *rope = nullptr, *h_state0 = nullptr;
  int n_prefix = -1;
};

}  // namespace

struct vla_ae {
  vla_ae_dims d{};
  int device = 0, num_sms = 148;
  bool fp8 = false;           // 8-bit weight codes with per-row scales (e4m3 or int8)
  int wq = 0;                 // weight format: 0 bf16, 1 e4m3, 2 int8
  int Ts = 0, Ntok = 0, NT = 0, Nt = 0, qd = 0, kd = 0, Lpad = 0;
  OpPlan op[4];
  size_t layer_wbytes = 0, layer_scales = 0;
  int attn_cs = 16;           // keys per attention sub-chunk (template argument)
  AttnParams attn_proto{};    // attention launch shape: S, span, nrb, Rpad, rpo, smem offsets
  // persistent engine
  bool loop_ok = false;       // planned (bf16, one n-tile, units fit the SMs)
  bool use_loop = false;      // selected (the engine the next capture uses)
  int engine_mode = VLA_AE_ENGINE_PER_OP;   // as set by vla_ae_set_engine
  int loop_cs = 16;           // attention sub-chunk of the persistent kernel
  LoopParams loop_proto{};    // plan: op shapes, smem layout, task lists, scratch
  size_t ctr_step = 0;        // counters per launch (layers x ctr_layer + abort word)
  unsigned* loop_dbg_ctr = nullptr;   // counter block of debug launches
  // device memory
  std::vector<void*> allocs;
  uint8_t* wpack = nullptr;
  float* wscale = nullptr;
  __nv_bfloat16 *w_in = nullptr, *b_in = nullptr, *w_st = nullptr, *b_st = nullptr, *w_out = nullptr,
                *b_out = nullptr, *w_ada = nullptr, *b_ada = nullptr, *w_fada = nullptr, *b_fada = nullptr;
  __nv_bfloat16 *kc = nullptr, *vct = nullptr, *act_x = nullptr, *act_o = nullptr, *act_m = nullptr,
                *noise_stage = nullptr, *state_stage = nullptr;
  __nv_bfloat16* q = nullptr;   // [B][nkv][Rpad][hd]: rows head_in_group * Ts + token, after RoPE
  float *h = nullptr, *ss = nullptr, *x = nullptr, *h_state0 = nullptr, *rope = nullptr, *out_stage = nullptr;
  double* temb = nullptr;
  unsigned* status = nullptr;
  size_t device_bytes = 0;
  int n_prefix = -1;
  // prefix slots: slot[front] is the one the loop reads (mirrored in kc / vct / rope / h_state0 /
  // n_prefix above); the other is the back slot vla_ae_set_prefix_next fills
  PrefixSlot slot[2];
  int front = 0;
  bool next_pending = false;
  cudaEvent_t next_ready = nullptr;
  int attn_P = -1;            // prefix length the per-op attention plan was made for
  // prefix K/V producer (vla_ae_attach_vlm_kv)
  bool vlm = false;
  int Hv = 0, NTp = 0, Ntp = 0;
  float vlm_eps = 1e-6f;
  OpPlan pkv;                 // the K/V GEMM over the prefix tokens (bf16)
  uint8_t* wpack_vlm = nullptr;
  float* vlm_gain = nullptr;  // [L][Hv]
  __nv_bfloat16* act_p = nullptr;   // operand tiles [Ntp][KBp][2][NTp][64]
  float *ss_p = nullptr, *rope_p = nullptr, *zeros_p = nullptr;
  cudaStream_t cap = nullptr;
  std::map<std::vector<double>, StepTables> tables;   // keyed by the time grid

  template <typename T>
  int alloc(T** p, size_t bytes) {
    void* v = nullptr;
    bytes = align_up(bytes ? bytes : 16, 256);
    CK(cudaMalloc(&v, bytes));
    allocs.push_back(v);
    CK(cudaMemset(v, 0, bytes));
    device_bytes += bytes;
    *p = reinterpret_cast<T*>(v);
    return VLA_AE_OK;
  }
  ~vla_ae() {
    for (auto& kv : tables)
      for (auto& g : kv.second.graphs) cudaGraphExecDestroy(g.second);
    if (next_ready) cudaEventDestroy(next_ready);
    for (void* p : allocs) cudaFree(p);
    if (cap) cudaStreamDestroy(cap);
  }
};

namespace {

// ------------------------------------------------------------------ launch helper
template <typename Kern, typename Arg>
cudaError_t launch(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x, bool pdl,
                   const Arg& arg) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  int n = 0;
  if (pdl) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attrs[n].id = cudaLaunchAttributeClusterDimension;
    attrs[n].val.clusterDim.x = cluster_x;
    attrs[n].val.clusterDim.y = 1;
    attrs[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, arg);
}

// Plain-argument kernel launch, optionally chained by programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_args(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                        Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// One CTA per SM for the whole launch: the cooperative attribute makes the launch fail instead of
// leaving CTAs unscheduled while others wait for them.
template <typename Kern, typename Arg>
cudaError_t launch_coop(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, const Arg& arg) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeCooperative;
  at.val.cooperative = 1;
  cfg.attrs = &at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, arg);
}

using GemmKernel = void (*)(const GemmParams);

// 64-wide k-blocks per packed weight tile of weight format wq (0 bf16, 1 e4m3, 2 int8, 3 int4)
int wq_kpt(int wq) { return wq == 3 ? 4 : wq ? 2 : 1; }
// fp32 scales per packed row of an op with K inputs: 1 (e4m3, int8), one per 128 inputs (int4)
int wq_scales_per_row(int wq, int K) { return wq == 3 ? ceil_div(K, 128) : 1; }

template <int EPI, bool NORM>
GemmKernel gemm_kernel_wq(int wq) {
  return wq == 3 ? gemm_stream_kernel<EPI, 3, NORM> : wq == 2 ? gemm_stream_kernel<EPI, 2, NORM>
         : wq == 1 ? gemm_stream_kernel<EPI, 1, NORM> : gemm_stream_kernel<EPI, 0, NORM>;
}
GemmKernel gemm_kernel_for(OpId id, int wq) {
  switch (id) {
    case OP_QKV: return gemm_kernel_wq<EPI_QKV, true>(wq);
    case OP_GU: return gemm_kernel_wq<EPI_SWIGLU, true>(wq);
    default: return gemm_kernel_wq<EPI_RESID, false>(wq);
  }
}

using AttnKernel = void (*)(const AttnParams);
template <int HD>
AttnKernel attn_kernel_cs(int cs) {
  switch (cs) {
    case 16: return attn_kernel<HD, 16>;
    case 32: return attn_kernel<HD, 32>;
    default: return attn_kernel<HD, 64>;
  }
}
AttnKernel attn_kernel_for(int hd, int cs) {
  switch (hd) {
    case 64: return attn_kernel_cs<64>(cs);
    case 128: return attn_kernel_cs<128>(cs);
    default: return attn_kernel_cs<256>(cs);
  }
}

// shared-memory layout of one GEMM op for a given (m-tiles per CTA, split, ring depth)
// kpt: 64-wide k-blocks per packed weight tile (1 bf16, 2 e4m3 / int8, 4 int4)
void gemm_layout(OpPlan& p, int NT, int kpt) {
  const bool fp8 = kpt > 1;
  const int nkt_max = ceil_div(p.KBt, p.S);
  const int nkb_max = std::min(nkt_max * kpt, p.KB);
  const size_t b_region = (size_t)2 * nkb_max * NT * 128;
  // split-K receive buffer [S][16 ceil(8 mpc / S)][NT + 4] fp32, over ring + operand
  const size_t red = (size_t)p.S * 16 * ceil_div(8 * p.mpc, p.S) * (NT + 4) * 4;
  size_t a_region = (size_t)p.stages * kTileBytes;
  if (a_region + b_region < red) a_region = red - b_region;
  a_region = align_up(a_region, 1024);
  const size_t conv = fp8 ? (size_t)kConvStages * kpt * kTileBytes : 0;
  p.off_b = (int)a_region;
  p.off_conv = (int)(a_region + align_up(b_region, 1024));
  p.off_bar = (int)(p.off_conv + conv);
  const size_t bar_bytes = 8 * (2 * p.stages + 2 + 2 * kConvStages) + 16;
  p.off_misc = (int)(p.off_bar + align_up(bar_bytes, 16));
  const int noct_max = ceil_div(p.mpc * 8, p.S);        // octets of 8 row pairs per rank
  const size_t misc = 4 * ((size_t)kMathThreads + NT + (size_t)NT * noct_max);
  p.off_vec = (int)(p.off_misc + align_up(misc, 16));
  p.smem = (int)(p.off_vec + (size_t)4 * 4 * p.mpc * 128 + 1024);   // + alignment slack
}

// one_wave: every cluster of the grid must be co-resident; else at least one cluster must fit
bool cluster_fits(GemmKernel kern, const OpPlan& p, int Nt, bool one_wave) {
  if (p.S == 1) return true;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.S, ceil_div(p.Mt, p.mpc), Nt);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = p.smem;
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeClusterDimension;
  a.val.clusterDim.x = p.S;
  a.val.clusterDim.y = 1;
  a.val.clusterDim.z = 1;
  cfg.attrs = &a;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return one_wave ? nclusters >= ceil_div(p.Mt, p.mpc) * Nt : nclusters >= 1;
}

// Choose m-tiles per CTA and the split so that one wave of CTAs covers the GPU with the
// fewest weight tiles per CTA, inside the shared-memory budget.  When no single-wave plan exists
// (many token tiles: large batches, the prefix producer), minimise an estimate of the launch's
// time instead: waves x per-CTA time, the latter in units of one resident tile's MMAs (~0.26 us):
// a fixed ~6 us per CTA (launch, operand, split-K exchange, epilogue), the tiles (slower when a
// shallow ring leaves L2 latency exposed) and the split-K push of the CTA's accumulators.
// Split / m-group / ring plan of one GEMM over Nt token tiles of NT rows with weight format wq.
int plan_gemm_shape(vla_ae* H, OpPlan& out, OpId id, int O, int K, int NT, int Nt, int wq) {
  const bool fp8 = wq != 0;
  OpPlan base;
  base.O = O;
  base.K = K;
  base.Mt = ceil_div(O, 128);
  base.KB = ceil_div(K, 64);
  const int kpt = wq_kpt(wq);
  base.KBt = ceil_div(K, 64 * kpt);
  base.wbytes = (size_t)base.Mt * base.KBt * kTileBytes;
  GemmKernel kern = gemm_kernel_for(id, wq);
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem));
  // every kernel of the loop asks for the same (maximum) shared-memory carveout, so SMs never
  // reconfigure between consecutive kernels and a dependent kernel's CTAs can co-reside
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  const int budget = kGemmSmemBudget;
  bool found = false;
  OpPlan best;
  long best_key = 0;
  for (int pass = 0; pass < 2 && !found; ++pass) {      // pass 1 allows more than one wave
    for (int mpc : {1, 2, 4}) {
      // TMEM: half of it (room for a dependent kernel's CTA beside this one), or all of it in
      // the several-wave pass
      if (mpc > base.Mt || mpc * 2 * NT > (pass == 0 ? 256 : 512)) continue;
      const int mg = ceil_div(base.Mt, mpc);
      for (int S = 1; S <= std::min(16, base.KBt); ++S) {
        const int ctas = mg * S * Nt;
        if (pass == 0 && ctas > H->num_sms) continue;   // pass 1: several waves (large batches)
        OpPlan p = base;
        p.mpc = mpc;
        p.S = S;
        const int tiles = mpc * ceil_div(base.KBt, S);
        // deepest ring inside the budget (at least 2 stages when there is more than one tile)
        p.stages = 1;
        gemm_layout(p, NT, kpt);
        for (int st = 2; st <= std::min(tiles, 8); ++st) {
          OpPlan t = p;
          t.stages = st;
          gemm_layout(t, NT, kpt);
          if (t.smem > (fp8 ? kMaxDynSmem : budget) && p.stages >= 2) break;
          if (t.smem > kMaxDynSmem) break;
          p = t;
        }
        if (p.smem > kMaxDynSmem) continue;
        const int over = p.smem > (fp8 ? kMaxDynSmem : budget) ? 1 : 0;
        // one wave: lexicographic (inside budget, fewest tiles per CTA, smallest split, fewest
        // m-tiles per CTA); several waves: estimated time first
        long cost = 0;
        if (pass == 1) {
          const int per_sm = (p.smem <= kMaxDynSmem / 2 - 1024 && mpc * 2 * NT <= 256) ? 2 : 1;
          const long waves = ceil_div(ctas, H->num_sms * per_sm);
          const double cta = 24.0 + tiles * std::max(1.0, 4.0 / p.stages) + (S > 1 ? mpc * NT / 48.0 : 0.0);
          cost = (long)(waves * cta * 100.0);
        }
        const long key = (long)over * 10000000000000L + cost * 1000000L + (long)tiles * 1000 + S * 10 + mpc;
        if (found && key >= best_key) continue;
        if (!cluster_fits(kern, p, Nt, pass == 0)) continue;
        best = p;
        best_key = key;
        found = true;
      }
    }
  }
  if (!found) return VLA_AE_EUNSUPPORTED;
  out = best;
  return VLA_AE_OK;
}

int plan_gemm(vla_ae* H, OpPlan& out, OpId id, int O, int K) {
  return plan_gemm_shape(H, out, id, O, K, H->NT, H->Nt, H->wq);
}

// Which source matrix row feeds packed row `pr` of op `id` (matrix: 0 q,1 k,2 v,3 o,4 g,5 u,6 d; -1 pad).
// QKV: each rotary pair (x_i, x_{i+hd/2}) of a q or k head becomes two adjacent packed rows so that
// the epilogue can rotate it locally; v rows keep their order.  Gate/up rows are interleaved so
// that SiLU(gate_j) * up_j is formed from two adjacent rows.
void packed_row_source(const vla_ae* H, OpId id, int pr, int* matrix, int* row) {
  const int hd = H->d.head_dim, half = hd / 2;
  *matrix = -1;
  *row = 0;
  switch (id) {
    case OP_QKV: {
      if (pr < H->qd + H->kd) {
        const bool isq = pr < H->qd;
        const int local = isq ? pr : pr - H->qd;
        const int head = local / hd, within = local % hd, i = within >> 1;
        *matrix = isq ? 0 : 1;
        *row = head * hd + i + ((within & 1) ? half : 0);
      } else if (pr < H->qd + 2 * H->kd) {
        *matrix = 2;
        *row = pr - H->qd - H->kd;
      }
      break;
    }
    case OP_O:
      if (pr < H->d.hidden) { *matrix = 3; *row = pr; }
      break;
    case OP_GU:
      if (pr < 2 * H->d.inter) { *matrix = (pr & 1) ? 5 : 4; *row = pr >> 1; }
      break;
    case OP_D:
      if (pr < H->d.hidden) { *matrix = 6; *row = pr; }
      break;
  }
}

int validate_dims(const vla_ae_dims* d) {
  if (!d) return VLA_AE_EINVAL;
  if (d->n_layers < 1 || d->hidden < 8 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->head_dim < 2 ||
      d->inter < 8 || d->t_emb_dim < 2 || d->action_dim < 1 || d->n_action_tokens < 1 || d->max_prefix < 0 ||
      d->batch < 1)
    return VLA_AE_EINVAL;
  if (d->has_state_token != 0 && d->has_state_token != 1) return VLA_AE_EINVAL;
  if (d->hidden % 8 || d->inter % 8 || d->t_emb_dim % 2 || d->n_q_heads % d->n_kv_heads) return VLA_AE_EINVAL;
  if (d->action_dim > kMaxAction) return VLA_AE_EINVAL;
  if ((long long)d->batch * (d->n_action_tokens + d->has_state_token) > 4096) return VLA_AE_EINVAL;
  if (!(d->rope_theta > 0.f) || !(d->rms_eps >= 0.f)) return VLA_AE_EINVAL;
  if (d->wtype != VLA_AE_BF16 && d->wtype != VLA_AE_FP8_E4M3 && d->wtype != VLA_AE_INT8 &&
      d->wtype != VLA_AE_INT4_G128)
    return VLA_AE_EINVAL;
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return VLA_AE_EUNSUPPORTED;
  return VLA_AE_OK;
}

// ------------------------------------------------------------------ attention plan
// Clusters: one per (sample, kv head, 64-row block of the head group's rep * Ts query rows).
// Keys are split over the cluster's CTAs in spans of a multiple of 16; the first choice fills
// the SMs with one CTA each, fewer CTAs per cluster are tried if a cluster does not fit.
int plan_attention(vla_ae* H, int P) {
  const vla_ae_dims& d = H->d;
  const int L = P + H->Ts;
  const int hd = d.head_dim;
  const int rep = d.n_q_heads / d.n_kv_heads;
  const int nrb = ceil_div(rep * H->Ts, kAttnRows);
  const int groups = nrb * d.n_kv_heads * d.batch;
  const int S0 = std::max(1, std::min({16, L, ceil_div(H->num_sms, groups)}));
  for (int Sc = S0; Sc >= 1; --Sc) {
    const int span = (int)align_up((size_t)ceil_div(L, Sc), 16);
    const int S = ceil_div(L, span);
    const int cs = span <= 16 ? 16 : span <= 32 ? 32 : 64;
    const int rpo = ceil_div(kAttnRows, S);
    AttnKernel kern = attn_kernel_for(hd, cs);
    CK(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem));
    CK(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
    AttnParams a{};
    size_t off = (size_t)attn_block_smem(hd, cs);   // q rows, K rows, V^T columns (bf16, padded rows)
    a.off_recv = (int)off;
    off += (size_t)S * rpo * (hd + 4) * 4;
    a.smem_bytes = (int)off;
    a.S = S;
    a.span = span;
    a.nrb = nrb;
    a.Rpad = nrb * kAttnRows;
    a.rpo = rpo;
    if (off > (size_t)kMaxDynSmem) continue;
    if (S > 1) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(S, nrb * d.n_kv_heads, d.batch);
      cfg.blockDim = dim3(kAttnThreads);
      cfg.dynamicSmemBytes = off;
      cudaLaunchAttribute at;
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = S;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      cfg.attrs = &at;
      cfg.numAttrs = 1;
      int ncl = 0;
      if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      if (ncl < 1) continue;
    }
    H->attn_cs = cs;
    H->attn_proto = a;
    return VLA_AE_OK;
  }
  return VLA_AE_EUNSUPPORTED;
}

// ------------------------------------------------------------------ persistent engine plan
using LoopKernel = void (*)(const LoopParams);
template <int HD>
LoopKernel loop_kernel_cs(int cs) {
  return cs <= 16 ? loop_kernel<HD, 16> : loop_kernel<HD, 32>;
}
LoopKernel loop_kernel_for(int hd, int cs) {
  switch (hd) {
    case 64: return loop_kernel_cs<64>(cs);
    case 128: return loop_kernel_cs<128>(cs);
    default: return loop_kernel_cs<256>(cs);
  }
}

// Work units and shared-memory layout of the persistent kernel.  Per GEMM: m-tiles per unit and
// split-K chosen so that every unit fits one SM (units <= SMs), the largest unit streams the
// fewest weight tiles, and its activation slice fits the operand buffer.  Attention: one unit
// per (sample, kv head, 64-row block, key span), spans planned for the longest prefix (a shorter
// prefix leaves trailing spans empty, which the merge weighs by zero).  Units are dealt to the
// CTAs round-robin, phase after phase, so each phase is spread over all SMs.  Leaves
// H->loop_ok false when the shape is outside the engine (fp8, more than one n-tile, ...).
int plan_loop(vla_ae* H) {
  const vla_ae_dims& d = H->d;
  H->loop_ok = false;
  if (H->fp8 || H->Nt != 1 || H->NT > 128 || d.hidden % 4 != 0) return VLA_AE_OK;
  const int G = H->num_sms, NT = H->NT, hd = d.head_dim;
  LoopParams lp{};
  const OpId ids[4] = {OP_QKV, OP_O, OP_GU, OP_D};
  // attention units
  const int rep = d.n_q_heads / d.n_kv_heads;
  const int nrb = ceil_div(rep * H->Ts, kAttnRows);
  const int groups = nrb * d.n_kv_heads * d.batch;
  const int Lmax = d.max_prefix + H->Ts;
  // key spans: up to 16 per block (at most two rounds of loads per merged value), as many as
  // the SMs allow; a span's own time grows with its length
  const int S0 = std::max(1, std::min({Lmax, 16, G / groups}));
  const int span = (int)align_up((size_t)ceil_div(Lmax, S0), 16);
  const int attn_S = ceil_div(Lmax, span);
  const int cs = span <= 16 ? 16 : 32;
  const size_t attn_bytes = (size_t)attn_block_smem(hd, cs);
  // GEMM units.  Latency model of one phase on the busiest CTA (microseconds, measured on the
  // persistent kernel): 1.5 per unit (accumulator hand-off, split wait, epilogue), 0.3 per
  // 128-row accumulator (partial store and reduction), 0.12 per weight tile already in the ring
  // (MMA issue), 0.36 per tile that must still stream when the phase starts (phase load above
  // the ring depth).  Search over operand-slice caps, which trade ring depth against split count.
  double best_cost = 1e30;
  int best_cfg[4][2] = {};
  for (size_t cap = 16 * 1024; cap <= 96 * 1024; cap += 8 * 1024) {
    int cfg[4][2], load[4], mpc_max = 1;
    double cost = 0.0;
    size_t slice_used = 0;
    bool ok = true;
    for (int i = 0; i < 4 && ok; ++i) {
      const OpPlan& q = H->op[ids[i]];
      double best = 1e30;
      cfg[i][0] = 0;
      for (int mpc : {1, 2, 4}) {
        if (mpc * 2 * NT > 256 || (mpc > 1 && mpc > q.Mt)) continue;
        const int ng = ceil_div(q.Mt, mpc);
        for (int S = 1; S <= q.KBt && ng * S <= 4 * G; ++S) {
          const int nk = ceil_div(q.KBt, S);
          if ((size_t)nk * 2 * NT * 128 > cap) continue;
          const int per_cta = ceil_div(ng * S, G);
          const double c = 0.12 * per_cta * std::min(mpc, q.Mt) * nk + 0.3 * per_cta * std::min(mpc, q.Mt) + 1.5 * per_cta;
          if (c < best - 1e-9) {
            best = c;
            cfg[i][0] = mpc;
            cfg[i][1] = S;
            load[i] = per_cta * std::min(mpc, q.Mt) * nk;
          }
        }
      }
      if (!cfg[i][0]) ok = false;
      if (!ok) break;
      mpc_max = std::max(mpc_max, cfg[i][0]);
      cost += best;
      slice_used = std::max(slice_used, (size_t)ceil_div(q.KBt, cfg[i][1]) * 2 * NT * 128);
    }
    if (!ok) continue;
    const size_t op_bytes = align_up(std::max(slice_used, attn_bytes), 1024);
    const size_t fixed = op_bytes + align_up((size_t)(kMathThreads + NT + NT * 32 * mpc_max) * 4, 16);
    const long long avail = (long long)kMaxDynSmem - 1024 - (long long)fixed - 1024;
    const int stages = (int)std::min<long long>(24, std::max<long long>(0, avail / kTileBytes));
    if (stages < 2) continue;
    for (int i = 0; i < 4; ++i) cost += 0.36 * std::max(0, load[i] - stages);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      std::memcpy(best_cfg, cfg, sizeof(cfg));
    }
  }
  if (best_cost >= 1e30) return VLA_AE_OK;
  int ctr = kPhases, mpc_max = 1, units_max = 1;
  size_t slice_used = 0;
  for (int i = 0; i < 4; ++i) {
    const OpPlan& q = H->op[ids[i]];
    LoopOp& o = lp.op[i];
    o.Mt = q.Mt;
    o.mpc = best_cfg[i][0];
    o.KBt = q.KBt;
    o.KB = q.KB;
    o.S = best_cfg[i][1];
    o.O = q.O;
    o.ngroups = ceil_div(q.Mt, o.mpc);
    o.parts_out = o.ngroups * o.S;
    o.ctr_base = ctr;
    o.woff = q.woff;
    ctr += o.ngroups;
    mpc_max = std::max(mpc_max, o.mpc);
    units_max = std::max(units_max, o.ngroups * o.S);
    slice_used = std::max(slice_used, (size_t)ceil_div(q.KBt, o.S) * 2 * NT * 128);
  }
  lp.attn_S = attn_S;
  lp.attn_span = span;
  lp.nrb = nrb;
  lp.attn_ctr_base = ctr;
  ctr += groups;
  lp.ctr_layer = (int)align_up((size_t)ctr, 32);
  // task lists
  std::vector<std::vector<uint32_t>> per(G);
  int cursor = 0;
  for (int ph = 0; ph < kPhases; ++ph) {
    const int units = ph == PH_ATTN ? groups * attn_S : lp.op[loop_phase_op(ph)].ngroups * lp.op[loop_phase_op(ph)].S;
    std::vector<char> has(G, 0);
    for (int u = 0; u < units; ++u, ++cursor) {
      per[cursor % G].push_back((uint32_t)ph << 24 | (uint32_t)u);
      has[cursor % G] = 1;
    }
    lp.phase_target[ph] = (int)std::count(has.begin(), has.end(), 1);
  }
  std::vector<uint32_t> tasks((size_t)G * kLoopMaxTasks, 0);
  std::vector<int> ntasks(G, 0);
  for (int c = 0; c < G; ++c) {
    if ((int)per[c].size() > kLoopMaxTasks) return VLA_AE_OK;
    ntasks[c] = (int)per[c].size();
    std::copy(per[c].begin(), per[c].end(), tasks.begin() + (size_t)c * kLoopMaxTasks);
  }
  // shared memory: ring | operand slice (or attention staging) | misc | barriers
  const size_t op_bytes = align_up(std::max(slice_used, attn_bytes), 1024);
  const size_t misc = (size_t)(kMathThreads + NT + NT * 32 * mpc_max) * 4;
  const size_t fixed = op_bytes + align_up(misc, 16);
  const size_t avail = (size_t)kMaxDynSmem - 1024 - fixed - 1024;
  const int stages = (int)std::min<size_t>(24, avail / kTileBytes);
  if (stages < 2) return VLA_AE_OK;
  size_t off = (size_t)stages * kTileBytes;
  lp.off_op = (int)off;
  off += op_bytes;
  lp.off_misc = (int)off;
  off += align_up(misc, 16);
  lp.off_bar = (int)off;
  off += (size_t)(2 * stages + 8) * 8 + 4 + kLoopMaxTasks * 4;
  lp.smem_bytes = (int)(off + 1024);
  lp.stages = stages;
  lp.mpc_max = mpc_max;
  lp.acc_cols = mpc_max * 2 * NT;
  lp.tmem_cols = 2 * lp.acc_cols <= 32 ? 32 : 2 * lp.acc_cols <= 64 ? 64 : 2 * lp.acc_cols <= 128 ? 128 : 2 * lp.acc_cols <= 256 ? 256 : 512;
  if (2 * lp.acc_cols > 512 || lp.smem_bytes > kMaxDynSmem) return VLA_AE_OK;
  LoopKernel kern = loop_kernel_for(hd, cs);
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lp.smem_bytes));
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  int per_sm = 0;
  CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLoopThreads, lp.smem_bytes));
  if (per_sm < 1) return VLA_AE_OK;
  // device buffers (fixed for the handle's lifetime)
  lp.gpart_unit = (size_t)128 * mpc_max * NT;
  int rc;
  if ((rc = H->alloc(&lp.gpart, (size_t)units_max * lp.gpart_unit * 4))) return rc;
  if ((rc = H->alloc(&lp.apart, (size_t)groups * attn_S * kAttnRows * (hd + 4) * 4))) return rc;
  uint32_t* dtasks = nullptr;
  int* dntasks = nullptr;
  if ((rc = H->alloc(&dtasks, tasks.size() * 4))) return rc;
  if ((rc = H->alloc(&dntasks, (size_t)G * 4))) return rc;
  CK(cudaMemcpy(dtasks, tasks.data(), tasks.size() * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dntasks, ntasks.data(), (size_t)G * 4, cudaMemcpyHostToDevice));
  lp.tasks = dtasks;
  lp.ntasks = dntasks;
  H->ctr_step = (size_t)d.n_layers * lp.ctr_layer + 32;
  if ((rc = H->alloc(&H->loop_dbg_ctr, H->ctr_step * 4))) return rc;
  H->loop_cs = cs;
  H->loop_proto = lp;
  H->loop_ok = true;   // available; the per-op engine stays the default (it measures faster)
  return VLA_AE_OK;
}

// ------------------------------------------------------------------ per-op launch
struct LayerPtrs {
  const float *shift_a, *scale_a, *gate_a, *shift_m, *scale_m, *gate_m;
};

LayerPtrs layer_mod(const vla_ae* H, const StepTables& T, int step, int layer) {
  const size_t Hd = H->d.hidden;
  const float* base = T.mod + ((size_t)step * H->d.n_layers + layer) * 6 * Hd;
  return {base, base + Hd, base + 2 * Hd, base + 3 * Hd, base + 4 * Hd, base + 5 * Hd};
}

void set_prefetch(const vla_ae* H, GemmParams& g, OpId id, int layer);

GemmParams gemm_common(const vla_ae* H, OpId id, int layer) {
  const OpPlan& p = H->op[id];
  GemmParams g{};
  set_prefetch(H, g, id, layer);
  g.w = H->wpack + (size_t)layer * H->layer_wbytes + p.woff;
  g.wscale = H->fp8 ? H->wscale + (size_t)layer * H->layer_scales + p.soff : nullptr;
  g.spr = wq_scales_per_row(H->wq, p.K);
  g.Mt = p.Mt;
  g.mpc = p.mpc;
  g.KBt = p.KBt;
  g.K = p.K;
  g.S = p.S;
  g.stages = p.stages;
  g.Ntok = H->Ntok;
  g.NT = H->NT;
  g.KB = p.KB;
  g.O = p.O;
  g.inv_h = 1.0f / (float)H->d.hidden;
  g.eps = H->d.rms_eps;
  g.status = H->status;
  g.off_b = p.off_b;
  g.off_conv = p.off_conv;
  g.off_bar = p.off_bar;
  g.off_misc = p.off_misc;
  g.off_vec = p.off_vec;
  g.smem_bytes = p.smem;
  return g;
}

// L2 prefetch target of a GEMM: the next GEMM of the loop (QKV -> o -> gate/up -> down -> next QKV)
void set_prefetch(const vla_ae* H, GemmParams& g, OpId id, int layer) {
  const OpId next = id == OP_QKV ? OP_O : id == OP_O ? OP_GU : id == OP_GU ? OP_D : OP_QKV;
  const int nl = id == OP_D ? (layer + 1) % H->d.n_layers : layer;
  g.pf_next = H->wpack + (size_t)nl * H->layer_wbytes + H->op[next].woff;
  g.pf_bytes = H->op[next].wbytes;
}

cudaError_t launch_gemm(const vla_ae* H, OpId id, const GemmParams& g, cudaStream_t st) {
  const OpPlan& p = H->op[id];
  return launch(gemm_kernel_for(id, H->wq), dim3(p.S, ceil_div(p.Mt, p.mpc), H->Nt), dim3(kGemmThreads), p.smem, st,
                p.S, true, g);
}

int ss_parts_of(const vla_ae* H, OpId id) { return ceil_div(H->op[id].Mt, H->op[id].mpc) * H->op[id].S; }

// Kernels of one DiT layer, in loop order.
enum LayerOp { LOP_QKV = 0, LOP_ATTN = 1, LOP_O = 2, LOP_GU = 3, LOP_D = 4 };

// One kernel of layer `layer` at step `step`.  `ss_in_parts`: partial sums of squares feeding
// the QKV kernel's RMSNorm (1 after the in-projection, those of the down GEMM otherwise).
cudaError_t enqueue_op(vla_ae* H, const StepTables& T, int step, int layer, int op, int ss_in_parts,
                       cudaStream_t st) {
  const vla_ae_dims& d = H->d;
  const LayerPtrs m = layer_mod(H, T, step, layer);
  const size_t cache = (size_t)layer * d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  const size_t cl = (size_t)step * d.n_layers + layer;
  switch (op) {
    case LOP_QKV: {  // (RMSNorm + modulate by linearity) QKV -> RoPE -> q, K/V caches
      GemmParams g = gemm_common(H, OP_QKV, layer);
      g.act = H->act_x;
      g.ss = H->ss;
      g.ss_parts = ss_in_parts;
      g.cshift = T.cq + cl * H->op[OP_QKV].Mt * 128;
      g.q_out = H->q;
      g.Rpad = H->attn_proto.Rpad;
      g.kc = H->kc + cache;
      g.vct = H->vct + cache;
      g.rope = H->rope;
      g.nq = d.n_q_heads;
      g.nkv = d.n_kv_heads;
      g.hd = d.head_dim;
      g.Ts = H->Ts;
      g.P = H->n_prefix;
      g.Lpad = H->Lpad;
      return launch_gemm(H, OP_QKV, g, st);
    }
    case LOP_ATTN: {  // attention over prefix + self
      AttnParams a = H->attn_proto;
      a.q = H->q;
      a.kc = H->kc + cache;
      a.vct = H->vct + cache;
      a.o_tiles = H->act_o;
      a.nq = d.n_q_heads;
      a.nkv = d.n_kv_heads;
      a.hd = d.head_dim;
      a.Ts = H->Ts;
      a.P = H->n_prefix;
      a.Lpad = H->Lpad;
      a.Ntok = H->Ntok;
      a.NT = H->NT;
      a.KBo = H->op[OP_O].KB;
      a.scale = (float)(1.0 / std::sqrt((double)d.head_dim));
      return launch(attn_kernel_for(d.head_dim, H->attn_cs), dim3(a.S, a.nrb * d.n_kv_heads, d.batch),
                    dim3(kAttnThreads), a.smem_bytes, st, a.S, true, a);
    }
    case LOP_O: {  // o-projection + gated residual; writes the gate/up operand h (1 + scale_m)
      GemmParams g = gemm_common(H, OP_O, layer);
      g.act = H->act_o;
      g.h = H->h;
      g.gate = m.gate_a;
      g.ss_out = H->ss;
      g.b_next = H->act_x;
      g.sc_next = m.scale_m;
      g.KBn = H->op[OP_GU].KB;
      return launch_gemm(H, OP_O, g, st);
    }
    case LOP_GU: {  // (RMSNorm + modulate by linearity) gate/up -> SwiGLU
      GemmParams g = gemm_common(H, OP_GU, layer);
      g.act = H->act_x;
      g.ss = H->ss;
      g.ss_parts = ss_parts_of(H, OP_O);
      g.cshift = T.cg + cl * H->op[OP_GU].Mt * 128;
      g.m_out = H->act_m;
      g.KBm = H->op[OP_D].KB;
      return launch_gemm(H, OP_GU, g, st);
    }
    default: {  // down-projection + gated residual; writes the next layer's QKV operand
      GemmParams g = gemm_common(H, OP_D, layer);
      g.act = H->act_m;
      g.h = H->h;
      g.gate = m.gate_m;
      g.ss_out = H->ss;
      if (layer + 1 < d.n_layers) {
        g.b_next = H->act_x;
        g.sc_next = layer_mod(H, T, step, layer + 1).scale_a;
        g.KBn = H->op[OP_QKV].KB;
      }
      return launch_gemm(H, OP_D, g, st);
    }
  }
}

cudaError_t enqueue_layer(vla_ae* H, const StepTables& T, int step, int layer, int ss_in_parts, cudaStream_t st,
                          const vla_ae_trace* trace) {
  const vla_ae_dims& d = H->d;
  const size_t cache = (size_t)layer * d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  cudaError_t e;
  if ((e = enqueue_op(H, T, step, layer, LOP_QKV, ss_in_parts, st)) != cudaSuccess) return e;
  if (trace && trace->q)
    q_trace_kernel<<<64, 256, 0, st>>>(H->q, trace->q, d.batch, H->Ts, d.n_q_heads, d.n_kv_heads, d.head_dim,
                                       H->attn_proto.Rpad);
  if (trace && trace->k && trace->v)
    self_kv_kernel<<<64, 256, 0, st>>>(H->kc + cache, H->vct + cache, trace->k, trace->v, d.batch, H->Ts,
                                       d.n_kv_heads, d.head_dim, H->n_prefix, H->Lpad);
  if ((e = enqueue_op(H, T, step, layer, LOP_ATTN, 0, st)) != cudaSuccess) return e;
  if (trace && trace->o) untile_kernel<<<64, 256, 0, st>>>(H->act_o, trace->o, H->Ntok, H->qd, H->NT, H->op[OP_O].KB);
  if ((e = enqueue_op(H, T, step, layer, LOP_O, 0, st)) != cudaSuccess) return e;
  if (trace && trace->h_attn)
    cudaMemcpyAsync(trace->h_attn, H->h, (size_t)H->Ntok * d.hidden * 4, cudaMemcpyDeviceToDevice, st);
  if ((e = enqueue_op(H, T, step, layer, LOP_GU, 0, st)) != cudaSuccess) return e;
  if (trace && trace->m) untile_kernel<<<64, 256, 0, st>>>(H->act_m, trace->m, H->Ntok, d.inter, H->NT, H->op[OP_D].KB);
  return enqueue_op(H, T, step, layer, LOP_D, 0, st);
}

TailParams tail_common(const vla_ae* H) {
  TailParams t{};
  t.h = H->h;
  t.ss = H->ss;
  t.ss_out = H->ss;
  t.w_out = H->w_out;
  t.b_out = H->b_out;
  t.w_in = H->w_in;
  t.b_in = H->b_in;
  t.h_state0 = H->h_state0;
  t.noise = H->noise_stage;
  t.x = H->x;
  t.b_out_tiles = H->act_x;
  t.NT = H->NT;
  t.KBh = H->op[OP_QKV].KB;
  t.eps = H->d.rms_eps;
  t.H = H->d.hidden;
  t.A = H->d.action_dim;
  t.T = H->d.n_action_tokens;
  t.Ts = H->Ts;
  t.has_state = H->d.has_state_token;
  t.Ntok = H->Ntok;
  return t;
}

cudaError_t launch_tail(const vla_ae* H, const TailParams& t, cudaStream_t st) {
  return launch(tail_kernel, dim3(H->Ntok), dim3(kTailThreads), 0, st, 1, true, t);
}

// The whole N-step loop (what the graph holds).
// sums-of-squares parts the last layer's down GEMM leaves for the tail kernel
int ss_parts_final(const vla_ae* H) { return H->use_loop ? H->loop_proto.op[3].parts_out : ss_parts_of(H, OP_D); }

// Persistent-engine launch over phases [(l0, ph0), (l1 - 1, ph1)) of step `step`; `ctr` is a
// zeroed counter block of ctr_step words.
cudaError_t launch_loop(const vla_ae* H, const StepTables& T, int step, unsigned* ctr, int l0, int ph0, int l1,
                        int ph1, int ss_first, cudaStream_t st) {
  const vla_ae_dims& d = H->d;
  LoopParams lp = H->loop_proto;
  lp.wpack = H->wpack;
  lp.layer_wbytes = H->layer_wbytes;
  lp.l0 = l0;
  lp.ph0 = ph0;
  lp.l1 = l1;
  lp.ph1 = ph1;
  lp.L = d.n_layers;
  lp.Ntok = H->Ntok;
  lp.NT = H->NT;
  lp.act_x = H->act_x;
  lp.act_o = H->act_o;
  lp.act_m = H->act_m;
  lp.h = H->h;
  lp.ss = H->ss;
  lp.ss_parts_first = ss_first;
  lp.q = H->q;
  lp.Rpad = H->attn_proto.Rpad;
  lp.kc = H->kc;
  lp.vct = H->vct;
  lp.cache_layer = (size_t)d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  lp.rope = H->rope;
  lp.nq = d.n_q_heads;
  lp.nkv = d.n_kv_heads;
  lp.hd = d.head_dim;
  lp.Ts = H->Ts;
  lp.P = H->n_prefix;
  lp.Lpad = H->Lpad;
  lp.B = d.batch;
  lp.cq_stride = H->op[OP_QKV].Mt * 128;
  lp.cg_stride = H->op[OP_GU].Mt * 128;
  lp.mod = T.mod + (size_t)step * d.n_layers * 6 * d.hidden;
  lp.cq = T.cq + (size_t)step * d.n_layers * lp.cq_stride;
  lp.cg = T.cg + (size_t)step * d.n_layers * lp.cg_stride;
  lp.inv_h = 1.0f / (float)d.hidden;
  lp.eps = d.rms_eps;
  lp.H = d.hidden;
  lp.scale = (float)(1.0 / std::sqrt((double)d.head_dim));
  lp.ctr = ctr;
  lp.status = H->status;
  return launch_coop(loop_kernel_for(d.head_dim, H->loop_cs), dim3(H->num_sms), dim3(kLoopThreads), lp.smem_bytes,
                     st, lp);
}

// Euler steps [k0, k1) of the loop of T.  The first step of the loop starts from the noise; a
// later segment starts from x as the previous segment left it (its in-projection runs here, so
// a segment uses its own prefix slot's state token).  The last step writes the actions.
cudaError_t enqueue_steps(vla_ae* H, const StepTables& T, int k0, int k1, cudaStream_t st) {
  const int N = T.steps, L = H->d.n_layers;
  cudaError_t e;
  if (H->use_loop && (e = cudaMemsetAsync(T.ctr + (size_t)k0 * H->ctr_step, 0,
                                          (size_t)(k1 - k0) * H->ctr_step * 4, st)) != cudaSuccess)
    return e;
  TailParams t0 = tail_common(H);
  t0.init_from_noise = k0 == 0;
  t0.do_in = 1;
  t0.sc_next = layer_mod(H, T, k0, 0).scale_a;
  if ((e = launch_tail(H, t0, st)) != cudaSuccess) return e;
  for (int k = k0; k < k1; ++k) {
    if (H->use_loop) {
      if ((e = launch_loop(H, T, k, T.ctr + (size_t)k * H->ctr_step, 0, 0, L, kPhases, 1, st)) != cudaSuccess) return e;
    } else {
      for (int l = 0; l < L; ++l)
        if ((e = enqueue_layer(H, T, k, l, l == 0 ? 1 : ss_parts_of(H, OP_D), st, nullptr)) != cudaSuccess) return e;
    }
    TailParams t = tail_common(H);
    t.ss_parts = ss_parts_final(H);
    t.shift_f = T.fmod + (size_t)k * 2 * H->d.hidden;
    t.scale_f = t.shift_f + H->d.hidden;
    t.dt = T.dt[k];
    t.do_out = 1;
    t.do_in = k + 1 < k1;
    if (t.do_in) t.sc_next = layer_mod(H, T, k + 1, 0).scale_a;
    t.out = k + 1 == N ? H->out_stage : nullptr;
    if ((e = launch_tail(H, t, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The tables of one time grid (t_0 > ... > t_n): adaLN modulation per (step, layer), the final
// modulation, the W . shift tables, the per-step dt and the persistent engine's counters.
// `uniform`: the grid of vla_ae_denoise (t_k = 1 - k/N), whose step is exactly -1/N.
int get_tables_grid(vla_ae* H, const std::vector<double>& grid, bool uniform, StepTables** out) {
  auto it = H->tables.find(grid);
  if (it != H->tables.end()) {
    *out = &it->second;
    return VLA_AE_OK;
  }
  const int steps = (int)grid.size() - 1;
  StepTables T;
  T.steps = steps;
  T.t = grid;
  T.dt.resize(steps);
  for (int k = 0; k < steps; ++k) T.dt[k] = uniform ? -1.0f / (float)steps : (float)(grid[k + 1] - grid[k]);
  const vla_ae_dims& d = H->d;
  const size_t Hd = d.hidden;
  int rc;
  if ((rc = H->alloc(&T.mod, (size_t)steps * d.n_layers * 6 * Hd * 4))) return rc;
  if ((rc = H->alloc(&T.fmod, (size_t)steps * 2 * Hd * 4))) return rc;
  double* c = nullptr;
  double* tdev = nullptr;
  CK(cudaMalloc(&c, (size_t)steps * d.t_emb_dim * sizeof(double)));
  CK(cudaMalloc(&tdev, (size_t)steps * sizeof(double)));
  CK(cudaMemcpy(tdev, grid.data(), (size_t)steps * sizeof(double), cudaMemcpyHostToDevice));
  temb_kernel<<<steps, 128, 0, H->cap>>>(tdev, c, d.t_emb_dim);
  for (int l = 0; l < d.n_layers; ++l) {
    const int rows = 6 * d.hidden;
    adaln_table_kernel<<<ceil_div(rows, 8), 256, 0, H->cap>>>(H->w_ada + (size_t)l * rows * d.t_emb_dim,
                                                                H->b_ada + (size_t)l * rows, c, rows, d.t_emb_dim,
                                                                steps, T.mod + (size_t)l * rows,
                                                                (size_t)d.n_layers * rows);
  }
  adaln_table_kernel<<<ceil_div(2 * d.hidden, 8), 256, 0, H->cap>>>(H->w_fada, H->b_fada, c, 2 * d.hidden,
                                                                     d.t_emb_dim, steps, T.fmod, 2 * Hd);
  CK(cudaGetLastError());
  // W . shift for the two normalised GEMMs of every (step, layer): RMSNorm's shift by linearity
  const size_t rq = (size_t)H->op[OP_QKV].Mt * 128, rg = (size_t)H->op[OP_GU].Mt * 128;
  if ((rc = H->alloc(&T.cq, (size_t)steps * d.n_layers * rq * 4))) return rc;
  if ((rc = H->alloc(&T.cg, (size_t)steps * d.n_layers * rg * 4))) return rc;
  if (H->loop_ok && (rc = H->alloc(&T.ctr, (size_t)steps * H->ctr_step * 4))) return rc;
  for (int l = 0; l < d.n_layers; ++l) {
    const uint8_t* wl = H->wpack + (size_t)l * H->layer_wbytes;
    const float* sl = H->fp8 ? H->wscale + (size_t)l * H->layer_scales : nullptr;
    const float* mod_l = T.mod + (size_t)l * 6 * Hd;
    const size_t mstep = (size_t)d.n_layers * 6 * Hd;
    const OpPlan& pq = H->op[OP_QKV];
    cshift_kernel<<<ceil_div((int)rq, 8), 256, 0, H->cap>>>(wl + pq.woff, sl ? sl + pq.soff : nullptr, (int)rq, pq.KBt,
                                                           pq.K, H->wq, wq_scales_per_row(H->wq, pq.K), mod_l + 0 * Hd, mstep, steps,
                                                           T.cq + (size_t)l * rq, (size_t)d.n_layers * rq);
    const OpPlan& pg = H->op[OP_GU];
    cshift_kernel<<<ceil_div((int)rg, 8), 256, 0, H->cap>>>(wl + pg.woff, sl ? sl + pg.soff : nullptr, (int)rg, pg.KBt,
                                                           pg.K, H->wq, wq_scales_per_row(H->wq, pg.K), mod_l + 3 * Hd, mstep, steps,
                                                           T.cg + (size_t)l * rg, (size_t)d.n_layers * rg);
  }
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(H->cap));
  CK(cudaFree(c));
  CK(cudaFree(tdev));
  auto res = H->tables.emplace(grid, T);
  *out = &res.first->second;
  return VLA_AE_OK;
}

std::vector<double> uniform_grid(int steps) {
  std::vector<double> g(steps + 1);
  for (int k = 0; k <= steps; ++k) g[k] = 1.0 - (double)k / (double)steps;
  return g;
}

int get_tables(vla_ae* H, int steps, StepTables** out) { return get_tables_grid(H, uniform_grid(steps), true, out); }

// Make prefix slot i the one the loop reads (the kernels take the mirrored fields), re-planning
// the per-op attention for its prefix length.
int use_slot(vla_ae* H, int i) {
  const PrefixSlot& sl = H->slot[i];
  H->kc = sl.kc;
  H->vct = sl.vct;
  H->rope = sl.rope;
  H->h_state0 = sl.h_state0;
  H->n_prefix = sl.n_prefix;
  if (sl.n_prefix >= 0 && sl.n_prefix != H->attn_P) {
    int rc = plan_attention(H, sl.n_prefix);
    if (rc) return rc;
    H->attn_P = sl.n_prefix;
  }
  return VLA_AE_OK;
}

// The graph of steps [k0, k1) of T on prefix slot `sl` (captured on first use).
int ensure_graph(vla_ae* H, StepTables* T, int k0, int k1, int sl, cudaGraphExec_t* out) {
  const std::array<int, 5> key = {k0, k1, sl, H->slot[sl].n_prefix, (int)H->use_loop};
  auto it = T->graphs.find(key);
  if (it != T->graphs.end()) {
    *out = it->second;
    return VLA_AE_OK;
  }
  int rc = use_slot(H, sl);
  if (rc) return rc;
  cudaGraph_t g = nullptr;
  cudaError_t e0 = cudaStreamBeginCapture(H->cap, cudaStreamCaptureModeThreadLocal);
  cudaError_t e = e0 == cudaSuccess ? enqueue_steps(H, *T, k0, k1, H->cap) : e0;
  cudaError_t e2 = e0 == cudaSuccess ? cudaStreamEndCapture(H->cap, &g) : e0;
  rc = use_slot(H, H->front);
  if (e != cudaSuccess || e2 != cudaSuccess) {
    std::fprintf(stderr, "vla_ae: graph capture failed: %s / %s\n", cudaGetErrorString(e), cudaGetErrorString(e2));
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return VLA_AE_ECUDA;
  }
  if (rc) {
    cudaGraphDestroy(g);
    return rc;
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  CK(ei);
  T->graphs.emplace(key, exec);
  *out = exec;
  return VLA_AE_OK;
}

// copy a bf16 blob (host or device) to a fresh device buffer owned by H
int upload_bf16(vla_ae* H, __nv_bfloat16** dst, const void* src, size_t n, int on_device) {
  int rc = H->alloc(dst, n * 2);
  if (rc) return rc;
  if (!src) return VLA_AE_EINVAL;
  CK(cudaMemcpy(*dst, src, n * 2, on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice));
  return VLA_AE_OK;
}

int pack_weights(vla_ae* H, const vla_ae_weights* w) {
  const vla_ae_dims& d = H->d;
  const int Hd = d.hidden, I = d.inter;
  const size_t sizes[7] = {(size_t)H->qd * Hd, (size_t)H->kd * Hd, (size_t)H->kd * Hd, (size_t)Hd * H->qd,
                           (size_t)I * Hd,     (size_t)I * Hd,     (size_t)Hd * I};
  const int ldk[7] = {Hd, Hd, Hd, H->qd, Hd, Hd, I};
  __nv_bfloat16* stage[7] = {};
  for (int i = 0; i < 7; ++i) CK(cudaMalloc(&stage[i], sizes[i] * 2));
  int maxrows = 0;
  for (int id = 0; id < 4; ++id) maxrows = std::max(maxrows, H->op[id].Mt * 128);
  const __nv_bfloat16** rowptr_dev = nullptr;
  CK(cudaMalloc(&rowptr_dev, (size_t)maxrows * sizeof(void*)));
  std::vector<const __nv_bfloat16*> rows(maxrows);
  const void* const* src_arrays[7] = {w->wq, w->wk, w->wv, w->wo, w->wg, w->wu, w->wd};
  int rc = VLA_AE_OK;
  for (int l = 0; l < d.n_layers && rc == VLA_AE_OK; ++l) {
    const __nv_bfloat16* src[7];
    for (int i = 0; i < 7; ++i) {
      if (!src_arrays[i] || !src_arrays[i][l]) { rc = VLA_AE_EINVAL; break; }
      if (w->on_device) {
        src[i] = reinterpret_cast<const __nv_bfloat16*>(src_arrays[i][l]);
      } else {
        CK(cudaMemcpy(stage[i], src_arrays[i][l], sizes[i] * 2, cudaMemcpyHostToDevice));
        src[i] = stage[i];
      }
    }
    if (rc) break;
    for (int id = 0; id < 4; ++id) {
      const OpPlan& p = H->op[id];
      for (int pr = 0; pr < p.Mt * 128; ++pr) {
        int mat, row;
        packed_row_source(H, (OpId)id, pr, &mat, &row);
        rows[pr] = mat < 0 ? nullptr : src[mat] + (size_t)row * ldk[mat];
      }
      CK(cudaMemcpy(rowptr_dev, rows.data(), (size_t)p.Mt * 128 * sizeof(void*), cudaMemcpyHostToDevice));
      uint8_t* dst = H->wpack + (size_t)l * H->layer_wbytes + p.woff;
      if (H->wq == 3) {
        quant_int4_kernel<<<ceil_div(p.Mt * 128, 8), 256>>>(rowptr_dev, p.K, p.Mt, p.KBt, dst,
                                                           H->wscale + (size_t)l * H->layer_scales + p.soff);
      } else if (H->wq == 2) {
        quant_int8_kernel<<<ceil_div(p.Mt * 128, 8), 256>>>(rowptr_dev, p.K, p.Mt, p.KBt, dst,
                                                           H->wscale + (size_t)l * H->layer_scales + p.soff);
      } else if (H->wq == 1) {
        quant_e4m3_kernel<<<ceil_div(p.Mt * 128, 8), 256>>>(rowptr_dev, p.K, p.Mt, p.KBt, dst,
                                                           H->wscale + (size_t)l * H->layer_scales + p.soff);
      } else {
        pack_bf16_kernel<<<1024, 256>>>(rowptr_dev, p.K, p.Mt, p.KB, dst);
      }
      CK(cudaGetLastError());
      CK(cudaDeviceSynchronize());   // rows[] and the staging buffers are reused
    }
  }
  for (int i = 0; i < 7; ++i) cudaFree(stage[i]);
  cudaFree(rowptr_dev);
  return rc;
}

int create_impl(const vla_ae_dims* dims, const vla_ae_weights* w, vla_ae* H) {
  int rc;
  H->d = *dims;
  const vla_ae_dims& d = H->d;
  H->wq = d.wtype == VLA_AE_FP8_E4M3 ? 1 : d.wtype == VLA_AE_INT8 ? 2 : d.wtype == VLA_AE_INT4_G128 ? 3 : 0;
  H->fp8 = H->wq != 0;
  CK(cudaGetDevice(&H->device));
  CK(cudaDeviceGetAttribute(&H->num_sms, cudaDevAttrMultiProcessorCount, H->device));
  int major = 0;
  CK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, H->device));
  if (major != 10) return VLA_AE_EUNSUPPORTED;
  CK(cudaStreamCreateWithFlags(&H->cap, cudaStreamNonBlocking));
  CK(cudaFuncSetAttribute(tail_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  H->Ts = d.n_action_tokens + d.has_state_token;
  H->Ntok = d.batch * H->Ts;
  // token tiles of at most 128 rows: the hi/lo operand pair then fits one MMA (N = 2 NT <= 256)
  // and a CTA's operand slice stays small enough for shared memory at any K
  H->Nt = ceil_div(H->Ntok, 128);
  H->NT = (int)align_up(ceil_div(H->Ntok, H->Nt), 32);
  H->qd = d.n_q_heads * d.head_dim;
  H->kd = d.n_kv_heads * d.head_dim;
  H->Lpad = (int)align_up((size_t)d.max_prefix + H->Ts, 8);
  if ((rc = plan_gemm(H, H->op[OP_QKV], OP_QKV, H->qd + 2 * H->kd, d.hidden))) return rc;
  if ((rc = plan_gemm(H, H->op[OP_O], OP_O, d.hidden, H->qd))) return rc;
  if ((rc = plan_gemm(H, H->op[OP_GU], OP_GU, 2 * d.inter, d.hidden))) return rc;
  if ((rc = plan_gemm(H, H->op[OP_D], OP_D, d.hidden, d.inter))) return rc;
  size_t woff = 0, soff = 0;
  for (int id = 0; id < 4; ++id) {
    H->op[id].woff = woff;
    H->op[id].soff = soff;
    woff += H->op[id].wbytes;
    soff += (size_t)H->op[id].Mt * 128 * wq_scales_per_row(H->wq, H->op[id].K);
  }
  H->layer_wbytes = woff;
  H->layer_scales = soff;
  if ((rc = plan_attention(H, d.max_prefix))) return rc;
  if ((rc = plan_loop(H))) return rc;

  const size_t L = d.n_layers, Hd = d.hidden, A = d.action_dim, B = d.batch;
  if ((rc = H->alloc(&H->wpack, L * H->layer_wbytes))) return rc;
  if (H->fp8 && (rc = H->alloc(&H->wscale, L * H->layer_scales * 4))) return rc;
  if ((rc = H->alloc(&H->status, 16))) return rc;
  const size_t cache = L * B * d.n_kv_heads * (size_t)H->Lpad * d.head_dim;
  if ((rc = H->alloc(&H->kc, cache * 2))) return rc;
  if ((rc = H->alloc(&H->vct, cache * 2))) return rc;
  if ((rc = H->alloc(&H->q, B * d.n_kv_heads * (size_t)H->attn_proto.Rpad * d.head_dim * 2))) return rc;
  if ((rc = H->alloc(&H->act_x, (size_t)H->Nt * H->op[OP_QKV].KB * 2 * H->NT * 64 * 2))) return rc;
  if ((rc = H->alloc(&H->act_o, (size_t)H->Nt * H->op[OP_O].KB * 2 * H->NT * 64 * 2))) return rc;
  if ((rc = H->alloc(&H->act_m, (size_t)H->Nt * H->op[OP_D].KB * 2 * H->NT * 64 * 2))) return rc;
  if ((rc = H->alloc(&H->noise_stage, B * d.n_action_tokens * A * 2))) return rc;
  if ((rc = H->alloc(&H->state_stage, B * A * 2))) return rc;
  if ((rc = H->alloc(&H->h, (size_t)H->Ntok * Hd * 4))) return rc;
  int parts = std::max({1, ss_parts_of(H, OP_O), ss_parts_of(H, OP_D)});
  if (H->loop_ok) parts = std::max({parts, H->loop_proto.op[1].parts_out, H->loop_proto.op[3].parts_out});
  if ((rc = H->alloc(&H->ss, (size_t)parts * H->Ntok * 4))) return rc;
  if ((rc = H->alloc(&H->x, B * d.n_action_tokens * A * 4))) return rc;
  if ((rc = H->alloc(&H->out_stage, B * d.n_action_tokens * A * 4))) return rc;
  if ((rc = H->alloc(&H->h_state0, B * Hd * 4))) return rc;
  if ((rc = H->alloc(&H->rope, (size_t)H->Ts * (d.head_dim / 2) * 8))) return rc;
  H->slot[0].kc = H->kc;
  H->slot[0].vct = H->vct;
  H->slot[0].rope = H->rope;
  H->slot[0].h_state0 = H->h_state0;
  H->attn_P = d.max_prefix;   // plan_attention ran for max_prefix above
  CK(cudaEventCreateWithFlags(&H->next_ready, cudaEventDisableTiming));

  if (!w) return VLA_AE_EINVAL;
  const int od = w->on_device;
  if (od) {  // device matrices are read in 16-byte vectors
    const void* const* arrays[7] = {w->wq, w->wk, w->wv, w->wo, w->wg, w->wu, w->wd};
    for (int i = 0; i < 7; ++i)
      for (size_t l = 0; arrays[i] && l < (size_t)d.n_layers; ++l)
        if (reinterpret_cast<uintptr_t>(arrays[i][l]) % 16) return VLA_AE_EINVAL;
  }
  if ((rc = upload_bf16(H, &H->w_in, w->w_in, Hd * A, od))) return rc;
  if ((rc = upload_bf16(H, &H->b_in, w->b_in, Hd, od))) return rc;
  if (d.has_state_token) {
    if ((rc = upload_bf16(H, &H->w_st, w->w_state, Hd * A, od))) return rc;
    if ((rc = upload_bf16(H, &H->b_st, w->b_state, Hd, od))) return rc;
  }
  if ((rc = upload_bf16(H, &H->w_out, w->w_out, A * Hd, od))) return rc;
  if ((rc = upload_bf16(H, &H->b_out, w->b_out, A, od))) return rc;
  if ((rc = upload_bf16(H, &H->w_fada, w->w_fada, 2 * Hd * d.t_emb_dim, od))) return rc;
  if ((rc = upload_bf16(H, &H->b_fada, w->b_fada, 2 * Hd, od))) return rc;
  if (!w->w_ada || !w->b_ada) return VLA_AE_EINVAL;
  if ((rc = H->alloc(&H->w_ada, L * 6 * Hd * d.t_emb_dim * 2))) return rc;
  if ((rc = H->alloc(&H->b_ada, L * 6 * Hd * 2))) return rc;
  for (size_t l = 0; l < L; ++l) {
    if (!w->w_ada[l] || !w->b_ada[l]) return VLA_AE_EINVAL;
    const cudaMemcpyKind kind = od ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    CK(cudaMemcpy(H->w_ada + l * 6 * Hd * d.t_emb_dim, w->w_ada[l], 6 * Hd * d.t_emb_dim * 2, kind));
    CK(cudaMemcpy(H->b_ada + l * 6 * Hd, w->b_ada[l], 6 * Hd * 2, kind));
  }
  if ((rc = pack_weights(H, w))) return rc;
  CK(cudaDeviceSynchronize());
  return VLA_AE_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* vla_ae_strerror(int code) {
  switch (code) {
    case VLA_AE_OK: return "ok";
    case VLA_AE_EINVAL: return "invalid argument";
    case VLA_AE_ENOMEM: return "out of device memory";
    case VLA_AE_ECUDA: return "CUDA error";
    case VLA_AE_ENOPREFIX: return "prefix not set";
    case VLA_AE_ETIMEOUT: return "device-side wait timed out";
    case VLA_AE_EUNSUPPORTED: return "unsupported configuration";
    default: return "unknown error";
  }
}

int vla_ae_create(const vla_ae_dims* dims, const vla_ae_weights* weights, vla_ae_t* out) {
  if (!out) return VLA_AE_EINVAL;
  *out = nullptr;
  int rc = validate_dims(dims);
  if (rc) return rc;
  if (!weights) return VLA_AE_EINVAL;
  auto H = std::make_unique<vla_ae>();
  rc = create_impl(dims, weights, H.get());
  if (rc) return rc;
  *out = H.release();
  return VLA_AE_OK;
}

void vla_ae_destroy(vla_ae_t h) {
  if (!h) return;
  cudaDeviceSynchronize();
  delete h;
}

// Lay a prefix out into slot i: K / V^T caches, projected state token, RoPE table of the self
// tokens at positions n_prefix + j.  Asynchronous on st.
static int write_prefix(vla_ae_t H, int i, const void* k, const void* v, int n_prefix, const void* state,
                        int on_device, cudaStream_t st) {
  const vla_ae_dims& d = H->d;
  PrefixSlot& sl = H->slot[i];
  const size_t n = (size_t)d.batch * d.n_layers * n_prefix * d.n_kv_heads * d.head_dim;
  if (n > 0) {
    const __nv_bfloat16 *kd = reinterpret_cast<const __nv_bfloat16*>(k), *vd = reinterpret_cast<const __nv_bfloat16*>(v);
    __nv_bfloat16 *kt = nullptr, *vt = nullptr;
    if (!on_device) {
      CK(cudaMallocAsync(&kt, n * 2, st));
      CK(cudaMallocAsync(&vt, n * 2, st));
      CK(cudaMemcpyAsync(kt, k, n * 2, cudaMemcpyHostToDevice, st));
      CK(cudaMemcpyAsync(vt, v, n * 2, cudaMemcpyHostToDevice, st));
      kd = kt;
      vd = vt;
    }
    prefix_layout_kernel<<<4 * H->num_sms, 256, 0, st>>>(kd, vd, sl.kc, sl.vct, d.batch, d.n_layers, n_prefix,
                                                         d.n_kv_heads, d.head_dim, H->Lpad);
    CK(cudaGetLastError());
    if (kt) CK(cudaFreeAsync(kt, st));
    if (vt) CK(cudaFreeAsync(vt, st));
  }
  if (d.has_state_token) {
    CK(cudaMemcpyAsync(H->state_stage, state, (size_t)d.batch * d.action_dim * 2,
                       on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, st));
    state_proj_kernel<<<dim3(ceil_div(d.hidden, 256), d.batch), 256, 0, st>>>(H->w_st, H->b_st, H->state_stage,
                                                                               sl.h_state0, d.hidden, d.action_dim);
  }
  rope_table_kernel<<<ceil_div(H->Ts * d.head_dim / 2, 256), 256, 0, st>>>(reinterpret_cast<float2*>(sl.rope), H->Ts,
                                                                           n_prefix, d.head_dim, (double)d.rope_theta);
  CK(cudaGetLastError());
  sl.n_prefix = n_prefix;
  return VLA_AE_OK;
}

int vla_ae_set_prefix(vla_ae_t H, const void* k, const void* v, int n_prefix, const void* state, int on_device,
                      void* stream) {
  if (!H || n_prefix < 0 || n_prefix > H->d.max_prefix) return VLA_AE_EINVAL;
  if (n_prefix > 0 && (!k || !v)) return VLA_AE_EINVAL;
  if (H->d.has_state_token && !state) return VLA_AE_EINVAL;
  int rc = write_prefix(H, H->front, k, v, n_prefix, state, on_device, reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  return use_slot(H, H->front);
}

int vla_ae_attach_vlm_kv(vla_ae_t H, const vla_ae_vlm_kv_weights* w) {
  if (!H || !w || w->hidden_vlm < 8 || w->hidden_vlm % 8 != 0 || !(w->rms_eps >= 0.f) || !w->wk || !w->wv || !w->gain)
    return VLA_AE_EINVAL;
  if (H->vlm) return VLA_AE_EINVAL;   // once per handle
  const vla_ae_dims& d = H->d;
  const int Hv = w->hidden_vlm, kd = H->kd, L = d.n_layers;
  // token tiling of the prefix rows (as for the action tokens: <= 128 rows per tile)
  const int ntok = d.batch * std::max(1, d.max_prefix);
  H->Ntp = ceil_div(ntok, 128);
  H->NTp = (int)align_up((size_t)ceil_div(ntok, H->Ntp), 32);
  int rc;
  if ((rc = plan_gemm_shape(H, H->pkv, OP_QKV, 2 * kd, Hv, H->NTp, H->Ntp, 0))) return rc;
  OpPlan& pk = H->pkv;
  if ((rc = H->alloc(&H->wpack_vlm, (size_t)L * pk.wbytes))) return rc;
  if ((rc = H->alloc(&H->vlm_gain, (size_t)L * Hv * 4))) return rc;
  if ((rc = H->alloc(&H->act_p, (size_t)H->Ntp * pk.KB * 2 * H->NTp * 64 * 2))) return rc;
  if ((rc = H->alloc(&H->ss_p, (size_t)H->Ntp * H->NTp * 4))) return rc;
  if ((rc = H->alloc(&H->rope_p, (size_t)std::max(1, d.max_prefix) * (d.head_dim / 2) * 8))) return rc;
  if ((rc = H->alloc(&H->zeros_p, (size_t)pk.Mt * 128 * 4))) return rc;
  // pack per layer: rows [0, kd) k with rotary pairs adjacent (as the QKV GEMM's k rows), then v
  const int hd = d.head_dim, half = hd / 2;
  __nv_bfloat16 *sk = nullptr, *sv = nullptr, *sg = nullptr;
  CK(cudaMalloc(&sk, (size_t)kd * Hv * 2));
  CK(cudaMalloc(&sv, (size_t)kd * Hv * 2));
  CK(cudaMalloc(&sg, (size_t)Hv * 2));
  const __nv_bfloat16** rowptr_dev = nullptr;
  CK(cudaMalloc(&rowptr_dev, (size_t)pk.Mt * 128 * sizeof(void*)));
  std::vector<const __nv_bfloat16*> rows((size_t)pk.Mt * 128, nullptr);
  const cudaMemcpyKind kind = w->on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  for (int l = 0; l < L; ++l) {
    if (!w->wk[l] || !w->wv[l] || !w->gain[l]) return VLA_AE_EINVAL;
    CK(cudaMemcpy(sk, w->wk[l], (size_t)kd * Hv * 2, kind));
    CK(cudaMemcpy(sv, w->wv[l], (size_t)kd * Hv * 2, kind));
    CK(cudaMemcpy(sg, w->gain[l], (size_t)Hv * 2, kind));
    for (int pr = 0; pr < pk.Mt * 128; ++pr) {
      const __nv_bfloat16* src = nullptr;
      if (pr < kd) {
        const int head = pr / hd, i = (pr % hd) / 2;
        src = sk + (size_t)(head * hd + i + (pr & 1) * half) * Hv;
      } else if (pr < 2 * kd) {
        src = sv + (size_t)(pr - kd) * Hv;
      }
      rows[pr] = src;
    }
    CK(cudaMemcpy(rowptr_dev, rows.data(), rows.size() * sizeof(void*), cudaMemcpyHostToDevice));
    pack_bf16_kernel<<<1024, 256>>>(rowptr_dev, Hv, pk.Mt, pk.KB, H->wpack_vlm + (size_t)l * pk.wbytes);
    bf16_to_f32_kernel<<<ceil_div(Hv, 256), 256>>>(sg, H->vlm_gain + (size_t)l * Hv, (size_t)Hv);
    CK(cudaGetLastError());
    CK(cudaDeviceSynchronize());   // the staging buffers are reused
  }
  cudaFree(sk);
  cudaFree(sv);
  cudaFree(sg);
  cudaFree(rowptr_dev);
  H->Hv = Hv;
  H->vlm_eps = w->rms_eps;
  H->vlm = true;
  return VLA_AE_OK;
}

int vla_ae_set_prefix_hidden(vla_ae_t H, const void* hidden, int n_prefix, const void* state, void* stream) {
  if (!H || !H->vlm || !hidden || n_prefix < 1 || n_prefix > H->d.max_prefix) return VLA_AE_EINVAL;
  if (H->d.has_state_token && !state) return VLA_AE_EINVAL;
  const vla_ae_dims& d = H->d;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const OpPlan& pk = H->pkv;
  const int ntok = d.batch * n_prefix, Nt = ceil_div(ntok, H->NTp);
  PrefixSlot& sl = H->slot[H->front];
  const size_t cache_layer = (size_t)d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  rope_table_kernel<<<ceil_div(n_prefix * d.head_dim / 2, 256), 256, 0, st>>>(reinterpret_cast<float2*>(H->rope_p),
                                                                              n_prefix, 0, d.head_dim,
                                                                              (double)d.rope_theta);
  for (int l = 0; l < d.n_layers; ++l) {
    CK(launch_args(prefix_operand_kernel, dim3(ntok), dim3(128), 0, st, l > 0,
                   reinterpret_cast<const __nv_bfloat16*>(hidden), (const float*)(H->vlm_gain + (size_t)l * H->Hv),
                   (int)d.n_layers, l, n_prefix, H->Hv, H->ss_p, H->act_p, H->NTp, pk.KB));
    GemmParams g{};
    g.w = H->wpack_vlm + (size_t)l * pk.wbytes;
    g.Mt = pk.Mt;
    g.mpc = pk.mpc;
    g.KBt = pk.KBt;
    g.K = pk.K;
    g.S = pk.S;
    g.stages = pk.stages;
    g.Ntok = ntok;
    g.NT = H->NTp;
    g.KB = pk.KB;
    g.O = pk.O;
    g.act = H->act_p;
    g.ss = H->ss_p;
    g.ss_parts = 1;
    g.cshift = H->zeros_p;
    g.inv_h = 1.0f / (float)H->Hv;
    g.eps = H->vlm_eps;
    g.kc = sl.kc + (size_t)l * cache_layer;
    g.vct = sl.vct + (size_t)l * cache_layer;
    g.rope = H->rope_p;
    g.nq = 0;   // K and V rows only
    g.nkv = d.n_kv_heads;
    g.hd = d.head_dim;
    g.Ts = n_prefix;   // token t -> sample t / P, position t % P
    g.P = 0;
    g.Lpad = H->Lpad;
    g.status = H->status;
    g.spr = 1;
    g.off_b = pk.off_b;
    g.off_conv = pk.off_conv;
    g.off_bar = pk.off_bar;
    g.off_misc = pk.off_misc;
    g.off_vec = pk.off_vec;
    g.smem_bytes = pk.smem;
    CK(launch(gemm_kernel_for(OP_QKV, 0), dim3(pk.S, ceil_div(pk.Mt, pk.mpc), Nt), dim3(kGemmThreads), pk.smem, st,
              pk.S, true, g));
  }
  // state token and the RoPE table of the self tokens at positions n_prefix + j
  if (d.has_state_token) {
    CK(cudaMemcpyAsync(H->state_stage, state, (size_t)d.batch * d.action_dim * 2, cudaMemcpyDeviceToDevice, st));
    state_proj_kernel<<<dim3(ceil_div(d.hidden, 256), d.batch), 256, 0, st>>>(H->w_st, H->b_st, H->state_stage,
                                                                               sl.h_state0, d.hidden, d.action_dim);
  }
  rope_table_kernel<<<ceil_div(H->Ts * d.head_dim / 2, 256), 256, 0, st>>>(reinterpret_cast<float2*>(sl.rope), H->Ts,
                                                                           n_prefix, d.head_dim, (double)d.rope_theta);
  CK(cudaGetLastError());
  sl.n_prefix = n_prefix;
  return use_slot(H, H->front);
}

int vla_ae_debug_prefix_kv(vla_ae_t H, int layer, float* k, float* v) {
  if (!H || !k || !v || layer < 0 || layer >= H->d.n_layers) return VLA_AE_EINVAL;
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  const vla_ae_dims& d = H->d;
  const size_t cache_layer = (size_t)d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  prefix_kv_readback_kernel<<<64, 256, 0, H->cap>>>(H->kc + layer * cache_layer, H->vct + layer * cache_layer, k, v,
                                                    d.batch, H->n_prefix, d.n_kv_heads, d.head_dim, H->Lpad);
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(H->cap));
  return VLA_AE_OK;
}

int vla_ae_set_prefix_next(vla_ae_t H, const void* k, const void* v, int n_prefix, const void* state, int on_device,
                           void* stream) {
  if (!H || n_prefix < 0 || n_prefix > H->d.max_prefix) return VLA_AE_EINVAL;
  if (n_prefix > 0 && (!k || !v)) return VLA_AE_EINVAL;
  if (H->d.has_state_token && !state) return VLA_AE_EINVAL;
  const int back = 1 - H->front;
  PrefixSlot& sl = H->slot[back];
  if (!sl.kc) {   // the back slot's buffers, on first use
    const vla_ae_dims& d = H->d;
    const size_t cache = (size_t)d.n_layers * d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
    int rc;
    if ((rc = H->alloc(&sl.kc, cache * 2))) return rc;
    if ((rc = H->alloc(&sl.vct, cache * 2))) return rc;
    if ((rc = H->alloc(&sl.h_state0, (size_t)d.batch * d.hidden * 4))) return rc;
    if ((rc = H->alloc(&sl.rope, (size_t)H->Ts * (d.head_dim / 2) * 8))) return rc;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int rc = write_prefix(H, back, k, v, n_prefix, state, on_device, st);
  if (rc) return rc;
  CK(cudaEventRecord(H->next_ready, st));
  H->next_pending = true;
  return VLA_AE_OK;
}

// VLA_AE_ENGINE_AUTO: on the first whole loop of T at the current prefix length, capture the loop
// with both engines and time a few replays of each on `st` (queued after the caller's noise copy,
// so they compute the very loop the caller asked for: every buffer a replay writes is rewritten by
// the launch that follows); the faster engine is kept for T and that prefix length.
static int auto_engine(vla_ae_t H, StepTables* T, cudaStream_t st) {
  const int key = H->slot[H->front].n_prefix;
  auto it = T->auto_loop.find(key);
  if (it != T->auto_loop.end()) {
    H->use_loop = it->second;
    return VLA_AE_OK;
  }
  if (!H->loop_ok) {
    H->use_loop = false;
    T->auto_loop.emplace(key, false);
    return VLA_AE_OK;
  }
  cudaEvent_t ev[2] = {nullptr, nullptr};
  if (cudaEventCreate(&ev[0]) != cudaSuccess || cudaEventCreate(&ev[1]) != cudaSuccess) {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
    cudaGetLastError();
    return VLA_AE_ECUDA;
  }
  float best = 0.f;
  bool pick = false;
  int rc = VLA_AE_OK;
  for (int lp = 0; lp < 2 && rc == VLA_AE_OK; ++lp) {
    H->use_loop = lp == 1;
    cudaGraphExec_t exec = nullptr;
    if ((rc = ensure_graph(H, T, 0, T->steps, H->front, &exec))) break;
    float ms = 0.f;
    if (cudaGraphLaunch(exec, st) != cudaSuccess || cudaEventRecord(ev[0], st) != cudaSuccess) rc = VLA_AE_ECUDA;
    for (int r = 0; r < 3 && rc == VLA_AE_OK; ++r)
      if (cudaGraphLaunch(exec, st) != cudaSuccess) rc = VLA_AE_ECUDA;
    if (rc == VLA_AE_OK && (cudaEventRecord(ev[1], st) != cudaSuccess || cudaEventSynchronize(ev[1]) != cudaSuccess ||
                            cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess))
      rc = VLA_AE_ECUDA;
    if (rc == VLA_AE_OK && (lp == 0 || ms < best)) {
      best = ms;
      pick = lp == 1;
    }
  }
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  if (rc) {
    cudaGetLastError();
    H->use_loop = false;
    return rc;
  }
  H->use_loop = pick;
  T->auto_loop.emplace(key, pick);
  return VLA_AE_OK;
}

static int denoise_tables(vla_ae_t H, StepTables* T, const void* noise, float* out, void* stream, bool host) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaGraphExec_t exec = nullptr;
  int rc;
  const vla_ae_dims& d = H->d;
  const size_t nx = (size_t)d.batch * d.n_action_tokens * d.action_dim;
  CK(cudaMemcpyAsync(H->noise_stage, noise, nx * 2, host ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st));
  if (H->engine_mode == VLA_AE_ENGINE_AUTO && (rc = auto_engine(H, T, st))) return rc;
  if ((rc = ensure_graph(H, T, 0, T->steps, H->front, &exec))) return rc;
  CK(cudaGraphLaunch(exec, st));
  CK(cudaMemcpyAsync(out, H->out_stage, nx * 4, host ? cudaMemcpyDeviceToHost : cudaMemcpyDeviceToDevice, st));
  return VLA_AE_OK;
}

static int denoise_common(vla_ae_t H, const void* noise, int steps, float* out, void* stream, bool host) {
  if (!H || !noise || !out || steps < 1) return VLA_AE_EINVAL;
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  StepTables* T = nullptr;
  int rc = get_tables(H, steps, &T);
  if (rc) return rc;
  return denoise_tables(H, T, noise, out, stream, host);
}

int vla_ae_denoise(vla_ae_t H, const void* noise, int steps, float* out, void* stream) {
  return denoise_common(H, noise, steps, out, stream, false);
}

int vla_ae_denoise_host(vla_ae_t H, const void* noise_host, int steps, float* out_host, void* stream) {
  return denoise_common(H, noise_host, steps, out_host, stream, true);
}

int vla_ae_denoise_stale(vla_ae_t H, const void* noise, int steps, int n_stale, float* out, void* stream) {
  if (!H || !noise || !out || steps < 1 || n_stale < 0 || n_stale > steps) return VLA_AE_EINVAL;
  if (H->n_prefix < 0 || !H->next_pending) return VLA_AE_ENOPREFIX;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  StepTables* T = nullptr;
  int rc = get_tables(H, steps, &T);
  if (rc) return rc;
  const int back = 1 - H->front;
  if (H->engine_mode == VLA_AE_ENGINE_AUTO) {   // the choice made for whole loops, if any
    auto it = T->auto_loop.find(H->slot[H->front].n_prefix);
    H->use_loop = it != T->auto_loop.end() && it->second;
  }
  cudaGraphExec_t ga = nullptr, gb = nullptr;
  if (n_stale > 0 && (rc = ensure_graph(H, T, 0, n_stale, H->front, &ga))) return rc;
  if (n_stale < steps && (rc = ensure_graph(H, T, n_stale, steps, back, &gb))) return rc;
  const vla_ae_dims& d = H->d;
  const size_t nx = (size_t)d.batch * d.n_action_tokens * d.action_dim;
  CK(cudaMemcpyAsync(H->noise_stage, noise, nx * 2, cudaMemcpyDeviceToDevice, st));
  if (ga) CK(cudaGraphLaunch(ga, st));
  CK(cudaStreamWaitEvent(st, H->next_ready, 0));   // the next prefix is laid out
  if (gb) CK(cudaGraphLaunch(gb, st));
  CK(cudaMemcpyAsync(out, H->out_stage, nx * 4, cudaMemcpyDeviceToDevice, st));
  H->front = back;   // the new prefix is the current one from now on
  H->next_pending = false;
  return use_slot(H, H->front);
}

int vla_ae_denoise_sched(vla_ae_t H, const void* noise, const float* t_grid, int n, float* out, void* stream) {
  if (!H || !noise || !out || !t_grid || n < 1 || n > VLA_AE_MAX_GRID_STEPS) return VLA_AE_EINVAL;
  std::vector<double> grid(n + 1);
  for (int k = 0; k <= n; ++k) {
    grid[k] = (double)t_grid[k];
    if (!std::isfinite(grid[k]) || (k > 0 && !(grid[k] < grid[k - 1]))) return VLA_AE_EINVAL;
  }
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  StepTables* T = nullptr;
  int rc = get_tables_grid(H, grid, false, &T);
  if (rc) return rc;
  return denoise_tables(H, T, noise, out, stream, false);
}

int vla_ae_status(vla_ae_t H) {
  if (!H) return VLA_AE_EINVAL;
  CK(cudaDeviceSynchronize());
  unsigned s = 0;
  CK(cudaMemcpy(&s, H->status, 4, cudaMemcpyDeviceToHost));
  CK(cudaMemset(H->status, 0, 4));
  return s ? VLA_AE_ETIMEOUT : VLA_AE_OK;
}

int vla_ae_query(vla_ae_t H, int what, int arg, long long* value) {
  if (!H || !value) return VLA_AE_EINVAL;
  const vla_ae_dims& d = H->d;
  switch (what) {
    case VLA_AE_Q_KERNELS_PER_LOOP:
      if (arg < 1) return VLA_AE_EINVAL;
      *value = 1 + (long long)arg * (H->use_loop ? 2LL : 5LL * d.n_layers + 1);
      return VLA_AE_OK;
    case VLA_AE_Q_ENGINE:
      *value = H->use_loop ? VLA_AE_ENGINE_PERSISTENT : VLA_AE_ENGINE_PER_OP;
      return VLA_AE_OK;
    case VLA_AE_Q_WEIGHT_BYTES: {
      long long b = 0;
      for (int id = 0; id < 4; ++id) b += (long long)H->op[id].wbytes;
      if (H->fp8) b += (long long)H->layer_scales * 4;
      *value = b * d.n_layers;
      return VLA_AE_OK;
    }
    case VLA_AE_Q_KV_BYTES:
      *value = 2LL * d.batch * d.n_layers * (long long)std::max(0, H->n_prefix) * d.n_kv_heads * d.head_dim * 2;
      return VLA_AE_OK;
    case VLA_AE_Q_DEVICE_BYTES:
      *value = (long long)H->device_bytes;
      return VLA_AE_OK;
    case VLA_AE_Q_OP_BYTES: {
      if (arg < 0 || arg > 4) return VLA_AE_EINVAL;
      if (arg == 1) {   // attention: prefix K + V of one layer (whole batch)
        *value = 2LL * d.batch * (long long)std::max(0, H->n_prefix) * d.n_kv_heads * d.head_dim * 2;
        return VLA_AE_OK;
      }
      const OpId id = arg == 0 ? OP_QKV : arg == 2 ? OP_O : arg == 3 ? OP_GU : OP_D;
      const long long ok = (long long)H->op[id].O * H->op[id].K;
      long long b = H->wq == 3 ? (ok + 1) / 2 : ok * (H->fp8 ? 1 : 2);
      if (H->fp8) b += 4LL * H->op[id].O * wq_scales_per_row(H->wq, H->op[id].K);
      *value = b;
      return VLA_AE_OK;
    }
    case VLA_AE_Q_SPLITS:
      *value = H->op[0].S | (H->op[1].S << 8) | (H->op[2].S << 16) | ((long long)H->op[3].S << 24);
      return VLA_AE_OK;
    default:
      return VLA_AE_EINVAL;
  }
}

int vla_ae_bench_op(vla_ae_t H, int op, int count, int steps, void* stream) {
  if (!H || op < 0 || op > 4 || count < 1 || steps < 1) return VLA_AE_EINVAL;
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  StepTables* T = nullptr;
  int rc = get_tables(H, steps, &T);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int parts = ss_parts_of(H, OP_D);
  for (int i = 0; i < count; ++i) CK(enqueue_op(H, *T, 0, i % H->d.n_layers, op, parts, st));
  return VLA_AE_OK;
}

int vla_ae_set_engine(vla_ae_t H, int engine) {
  if (!H || (engine != VLA_AE_ENGINE_PER_OP && engine != VLA_AE_ENGINE_PERSISTENT && engine != VLA_AE_ENGINE_AUTO))
    return VLA_AE_EINVAL;
  if (engine == VLA_AE_ENGINE_PERSISTENT && !H->loop_ok) return VLA_AE_EUNSUPPORTED;
  H->engine_mode = engine;
  // graphs of the other engine re-capture on their next use; AUTO keeps the current engine until
  // its first whole loop decides
  if (engine != VLA_AE_ENGINE_AUTO) H->use_loop = engine == VLA_AE_ENGINE_PERSISTENT;
  return VLA_AE_OK;
}

int vla_ae_debug_wait_probe(vla_ae_t H, unsigned attempts) {
  if (!H || attempts == 0 || attempts > (1u << 20)) return VLA_AE_EINVAL;
  wait_probe_kernel<<<1, 32, 0, H->cap>>>(attempts, H->status);
  CK(cudaGetLastError());
  CK(cudaStreamSynchronize(H->cap));
  return VLA_AE_OK;
}

int vla_ae_debug_layer(vla_ae_t H, int layer, int step, int steps, const float* h_in, float* h_out,
                       const vla_ae_trace* trace) {
  if (!H || !h_in || !h_out || layer < 0 || layer >= H->d.n_layers || steps < 1 || step < 0 || step >= steps)
    return VLA_AE_EINVAL;
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  StepTables* T = nullptr;
  int rc = get_tables(H, steps, &T);
  if (rc) return rc;
  const size_t nh = (size_t)H->Ntok * H->d.hidden;
  cudaStream_t st = H->cap;
  CK(cudaMemcpyAsync(H->h, h_in, nh * 4, cudaMemcpyDeviceToDevice, st));
  // sums of squares of h_in (a single part) and the QKV operand h (1 + scale_attn)
  row_operand_kernel<<<H->Ntok, 256, 0, st>>>(H->h, H->ss, H->act_x, layer_mod(H, *T, step, layer).scale_a,
                                              H->d.hidden, H->NT, H->op[OP_QKV].KB);
  CK(cudaGetLastError());
  if (H->use_loop) {
    // persistent engine: the layer in one launch, or in two (through the o-projection, then the
    // MLP) when intermediates are traced
    const vla_ae_dims& d = H->d;
    const size_t cache = (size_t)layer * d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
    const bool split = trace != nullptr;
    CK(cudaMemsetAsync(H->loop_dbg_ctr, 0, H->ctr_step * 4, st));
    CK(launch_loop(H, *T, step, H->loop_dbg_ctr, layer, 0, layer + 1, split ? (int)PH_GU : (int)kPhases, 1, st));
    if (split) {
      if (trace->q)
        q_trace_kernel<<<64, 256, 0, st>>>(H->q, trace->q, d.batch, H->Ts, d.n_q_heads, d.n_kv_heads, d.head_dim,
                                           H->attn_proto.Rpad);
      if (trace->k && trace->v)
        self_kv_kernel<<<64, 256, 0, st>>>(H->kc + cache, H->vct + cache, trace->k, trace->v, d.batch, H->Ts,
                                           d.n_kv_heads, d.head_dim, H->n_prefix, H->Lpad);
      if (trace->o) untile_kernel<<<64, 256, 0, st>>>(H->act_o, trace->o, H->Ntok, H->qd, H->NT, H->op[OP_O].KB);
      if (trace->h_attn) CK(cudaMemcpyAsync(trace->h_attn, H->h, nh * 4, cudaMemcpyDeviceToDevice, st));
      CK(cudaMemsetAsync(H->loop_dbg_ctr, 0, H->ctr_step * 4, st));
      CK(launch_loop(H, *T, step, H->loop_dbg_ctr, layer, PH_GU, layer + 1, kPhases, 1, st));
      if (trace->m) untile_kernel<<<64, 256, 0, st>>>(H->act_m, trace->m, H->Ntok, d.inter, H->NT, H->op[OP_D].KB);
    }
    CK(cudaGetLastError());
  } else {
    CK(enqueue_layer(H, *T, step, layer, 1, st, trace));
  }
  CK(cudaMemcpyAsync(h_out, H->h, nh * 4, cudaMemcpyDeviceToDevice, st));
  CK(cudaStreamSynchronize(st));
  return VLA_AE_OK;
}

int vla_ae_debug_velocity(vla_ae_t H, int step, int steps, const float* x, float* v) {
  if (!H || !x || !v || steps < 1 || step < 0 || step >= steps) return VLA_AE_EINVAL;
  if (H->n_prefix < 0) return VLA_AE_ENOPREFIX;
  StepTables* T = nullptr;
  int rc = get_tables(H, steps, &T);
  if (rc) return rc;
  const vla_ae_dims& d = H->d;
  cudaStream_t st = H->cap;
  const size_t nx = (size_t)d.batch * d.n_action_tokens * d.action_dim;
  CK(cudaMemcpyAsync(H->x, x, nx * 4, cudaMemcpyDeviceToDevice, st));
  TailParams t0 = tail_common(H);
  t0.do_in = 1;
  t0.sc_next = layer_mod(H, *T, step, 0).scale_a;
  CK(launch_tail(H, t0, st));
  if (H->use_loop) {
    CK(cudaMemsetAsync(H->loop_dbg_ctr, 0, H->ctr_step * 4, st));
    CK(launch_loop(H, *T, step, H->loop_dbg_ctr, 0, 0, d.n_layers, kPhases, 1, st));
  } else {
    for (int l = 0; l < d.n_layers; ++l)
      CK(enqueue_layer(H, *T, step, l, l == 0 ? 1 : ss_parts_of(H, OP_D), st, nullptr));
  }
  TailParams t = tail_common(H);
  t.ss_parts = ss_parts_final(H);
  t.shift_f = T->fmod + (size_t)step * 2 * d.hidden;
  t.scale_f = t.shift_f + d.hidden;
  t.dt = 0.f;
  t.do_out = 1;
  t.v_out = v;
  CK(launch_tail(H, t, st));
  CK(cudaStreamSynchronize(st));
  return VLA_AE_OK;
}

int vla_ae_debug_weight(vla_ae_t H, int layer, int which, void* w_host, float* scales_host) {
  if (!H || !w_host || layer < 0 || layer >= H->d.n_layers || which < 0 || which > 6) return VLA_AE_EINVAL;
  const OpId id = which <= 2 ? OP_QKV : which == 3 ? OP_O : which <= 5 ? OP_GU : OP_D;
  const OpPlan& p = H->op[id];
  std::vector<uint8_t> blob(p.wbytes);
  CK(cudaMemcpy(blob.data(), H->wpack + (size_t)layer * H->layer_wbytes + p.woff, p.wbytes, cudaMemcpyDeviceToHost));
  std::vector<float> sc;
  const int spr = wq_scales_per_row(H->wq, p.K);
  if (H->fp8) {
    sc.resize((size_t)p.Mt * 128 * spr);
    CK(cudaMemcpy(sc.data(), H->wscale + (size_t)layer * H->layer_scales + p.soff, sc.size() * 4,
                  cudaMemcpyDeviceToHost));
  }
  const int K = p.K;
  for (int pr = 0; pr < p.Mt * 128; ++pr) {
    int mat, row;
    packed_row_source(H, id, pr, &mat, &row);
    if (mat != which) continue;
    const int mt = pr / 128, r = pr % 128;
    for (int k = 0; k < K; ++k) {
      if (H->wq == 3) {   // int4: two codes per byte (low nibble first), returned one per byte
        const size_t tile = (size_t)mt * p.KBt + k / 256;
        const int kk = k % 256;
        const size_t byte = tile * kTileBytes + sw128_chunk_byte(r, kk / 32) + (kk % 32) / 2;
        const int nib = (blob[byte] >> (4 * (kk & 1))) & 0xF;
        reinterpret_cast<int8_t*>(w_host)[(size_t)row * K + k] = (int8_t)((nib ^ 8) - 8);
      } else if (H->fp8) {
        const size_t tile = (size_t)mt * p.KBt + k / 128;
        const int kk = k % 128;
        const size_t byte = tile * kTileBytes + sw128_chunk_byte(r, kk / 16) + (kk % 16);
        reinterpret_cast<uint8_t*>(w_host)[(size_t)row * K + k] = blob[byte];
      } else {
        const size_t tile = (size_t)mt * p.KBt + k / 64;
        const size_t elem = tile * (kTileBytes / 2) + sw128_elem_offset(r, k % 64);
        reinterpret_cast<uint16_t*>(w_host)[(size_t)row * K + k] = reinterpret_cast<const uint16_t*>(blob.data())[elem];
      }
    }
    if (H->fp8 && scales_host)
      for (int g = 0; g < spr; ++g) scales_host[(size_t)row * spr + g] = sc[(size_t)pr * spr + g];
  }
  return VLA_AE_OK;
}

}  // extern "C"

// ====================================================================== allocation-free prefix upload
// Some callers cannot allocate device memory while they run: a robot control loop that must not
// take the allocator's unbounded latency every cycle, or code that runs while a CUDA graph is
// being captured on the device (an allocation there is not allowed).  vla_ae_set_prefix with
// host pointers stages the prefix through cudaMallocAsync'd buffers; vla_ae_set_prefix_static
// stages it instead, one layer at a time, through this fixed array compiled into the library.
// Every GPU that loads the library holds the array until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // VLA_AE_STATIC_SCRATCH_BYTES
static __device__ __align__(256) uint8_t g_prefix_scratch[kStaticScratchBytes];

// One layer of the prefix, read from the static staging array: K, V [B][P][nkv][hd] ->
// the layer's K cache [B][nkv][Lpad][hd] and V^T cache [B][nkv][hd][Lpad].
__global__ void prefix_layout_static_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                            __nv_bfloat16* kc, __nv_bfloat16* vct, int B, int P, int nkv, int hd,
                                            int Lpad) {
  const size_t total = (size_t)B * P * nkv * hd;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int d = (int)(e % hd);
    size_t r = e / hd;
    const int g = (int)(r % nkv);
    r /= nkv;
    const int pp = (int)(r % P);
    const int b = (int)(r / P);
    const size_t cache = (size_t)b * nkv + g;
    kc[(cache * Lpad + pp) * hd + d] = k[e];
    vct[(cache * hd + d) * Lpad + pp] = v[e];
  }
}

std::mutex g_scratch_mutex;
void* g_scratch_ptr[64] = {};   // device address of g_prefix_scratch, per device, set on first use

int static_scratch(int device, uint8_t** out) {
  if (device < 0 || device >= 64) return VLA_AE_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[device]) {
    void* p = nullptr;
    // in host code the array's name only stands for the symbol: ask the runtime for its address
    cudaError_t e = cudaGetSymbolAddress(&p, g_prefix_scratch);
    if (e != cudaSuccess || !p) {
      std::fprintf(stderr, "vla_ae_set_prefix_static: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
      return VLA_AE_ECUDA;
    }
    g_scratch_ptr[device] = p;
  }
  *out = reinterpret_cast<uint8_t*>(g_scratch_ptr[device]);
  return VLA_AE_OK;
}

}  // namespace

extern "C" int vla_ae_set_prefix_static(vla_ae_t H, const void* k, const void* v, int n_prefix, const void* state,
                                        void* stream) {
  if (!H || n_prefix < 0 || n_prefix > H->d.max_prefix) return VLA_AE_EINVAL;
  if (n_prefix > 0 && (!k || !v)) return VLA_AE_EINVAL;
  if (H->d.has_state_token && !state) return VLA_AE_EINVAL;
  const vla_ae_dims& d = H->d;
  const size_t per_sample = (size_t)n_prefix * d.n_kv_heads * d.head_dim;   // elements per (sample, layer)
  const size_t layer_bytes = 2 * (size_t)d.batch * per_sample * 2;         // K and V of one layer, bf16
  if (layer_bytes > kStaticScratchBytes) {
    std::fprintf(stderr,
                 "vla_ae_set_prefix_static: one layer of prefix K+V needs %zu bytes, more than the %zu-byte "
                 "static staging array (batch * n_prefix * n_kv_heads * head_dim * 4 must be <= %zu)\n",
                 layer_bytes, kStaticScratchBytes, kStaticScratchBytes);
    return VLA_AE_EINVAL;
  }
  uint8_t* scratch = nullptr;
  int rc = static_scratch(H->device, &scratch);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(scratch);
  __nv_bfloat16* vs = ks + (size_t)d.batch * per_sample;
  const size_t cache_layer = (size_t)d.batch * d.n_kv_heads * H->Lpad * d.head_dim;
  for (int l = 0; l < d.n_layers && per_sample > 0; ++l) {
    // stream order keeps this layer's copies behind the previous layer's kernel (the array is reused)
    for (int b = 0; b < d.batch; ++b) {
      const size_t src = ((size_t)b * d.n_layers + l) * per_sample * 2;   // bytes into [B][L][P][nkv][hd]
      CK(cudaMemcpyAsync(ks + (size_t)b * per_sample, reinterpret_cast<const uint8_t*>(k) + src, per_sample * 2,
                         cudaMemcpyHostToDevice, st));
      CK(cudaMemcpyAsync(vs + (size_t)b * per_sample, reinterpret_cast<const uint8_t*>(v) + src, per_sample * 2,
                         cudaMemcpyHostToDevice, st));
    }
    prefix_layout_static_kernel<<<4 * H->num_sms, 256, 0, st>>>(ks, vs, H->kc + l * cache_layer, H->vct + l * cache_layer,
                                                                d.batch, n_prefix, d.n_kv_heads, d.head_dim, H->Lpad);
    CK(cudaGetLastError());
  }
  if (d.has_state_token) {
    CK(cudaMemcpyAsync(H->state_stage, state, (size_t)d.batch * d.action_dim * 2, cudaMemcpyHostToDevice, st));
    state_proj_kernel<<<dim3(ceil_div(d.hidden, 256), d.batch), 256, 0, st>>>(H->w_st, H->b_st, H->state_stage,
                                                                               H->h_state0, d.hidden, d.action_dim);
  }
  rope_table_kernel<<<ceil_div(H->Ts * d.head_dim / 2, 256), 256, 0, st>>>(reinterpret_cast<float2*>(H->rope), H->Ts,
                                                                           n_prefix, d.head_dim, (double)d.rope_theta);
  CK(cudaGetLastError());
  H->slot[H->front].n_prefix = n_prefix;   // (H->kc ... mirror the front slot's buffers)
  return use_slot(H, H->front);
}
