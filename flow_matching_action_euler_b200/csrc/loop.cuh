// Persistent layer-loop kernel: one launch runs every layer of one Euler step of the action
// expert ("VLA-Perf" section 4: batch-1 denoising is a chain of small, memory-bound kernels, so
// kernel boundaries and their tails, not the weight stream, set the pace).
//
// One CTA per SM stays resident for the whole step.  Each CTA owns a fixed list of work units
// per layer, sorted by phase (QKV, attention, o-proj, gate/up, down); the same list repeats for
// every layer.  Roles inside a CTA:
//
//  * warp 0, producer: streams the weight tiles of all its GEMM units of all layers, in order,
//    through a ring of 16 KB shared-memory stages with 1-D bulk copies.  It never waits on
//    activations, so HBM keeps streaming across phase and layer boundaries while the MMA side
//    waits on data dependencies.
//  * warp 1, MMA issuer: per GEMM unit it waits until the phase that produces its operand is
//    complete (a grid-scope counter, acquire), bulk-copies its K-slice of the hi/lo activation
//    tiles, and issues one tcgen05.mma per K step into one of two TMEM accumulators.
//  * warps 2-5, math: per phase, pass A writes every unit's fp32 split-K partial to global
//    memory (and computes attention partials); pass B waits for all splits of the unit, reduces
//    the rows this split owns in rank order (deterministic) and runs the fused epilogue
//    (RMSNorm scale by linearity, RoPE + q/K/V-cache writes, gated residual + next operand,
//    SwiGLU); then one release increment of the phase counter.  Because every CTA finishes pass A
//    of a phase before any of its pass-B waits, no wait can close a cycle.
//
// The epilogue arithmetic is the same as the per-op GEMM kernel's (gemm.cuh).  Every wait is
// bounded by the global timer and by a per-launch abort word: a wait that runs out flags the
// status word, raises the abort word so all other waits return at once, and the kernel drains its
// own copies and frees its TMEM before returning.
#pragma once
#include "attention.cuh"
#include "gemm.cuh"

namespace vla {

constexpr int kLoopThreads = 192;
constexpr int kLoopMaxTasks = 16;           // work units per CTA per layer
constexpr uint64_t kLoopWaitNs = 1000000000ull;   // 1 s: far above any legitimate wait in a step
enum LoopPhase : int { PH_QKV = 0, PH_ATTN = 1, PH_O = 2, PH_GU = 3, PH_D = 4, kPhases = 5 };

struct LoopOp {        // one GEMM of the layer (the shape is the same in every layer)
  int Mt, mpc, KBt, KB, S, O;
  int ngroups;          // ceil(Mt / mpc) groups of m-tiles; unit = group * S + split
  int parts_out;        // RESID: sums-of-squares parts written (= ngroups * S)
  int ctr_base;         // first per-group counter inside a layer's counter block
  size_t woff;          // byte offset of the op's tiles inside one layer's packed weights
};

struct LoopParams {
  const uint8_t* wpack;
  size_t layer_wbytes;
  LoopOp op[4];         // QKV, O, GU, D
  int l0, l1, L;        // layers run by this launch, layers of the model
  int ph0, ph1;         // first phase of layer l0, end phase of layer l1 - 1 (0 and 5 for whole layers)
  int stages;           // weight ring depth
  int Ntok, NT;
  __nv_bfloat16 *act_x, *act_o, *act_m;   // operand tiles [1][KB][2][NT][64]
  float* h;             // residual [Ntok][H]
  float* ss;            // partial sums of squares [parts][Ntok]
  int ss_parts_first;   // parts feeding the first layer's QKV
  __nv_bfloat16* q;     // [B][nkv][Rpad][hd]
  int Rpad;
  __nv_bfloat16 *kc, *vct;   // caches of layer 0; layer l adds l * cache_layer elements
  size_t cache_layer;
  const float* rope;    // [Ts][hd/2][2]
  int nq, nkv, hd, Ts, P, Lpad, B;
  const float* mod;     // this step's adaLN table [L][6][H]
  const float* cq;      // this step's W_qkv . shift_a [L][cq_stride]
  const float* cg;      // this step's W_gu . shift_m [L][cg_stride]
  int cq_stride, cg_stride;
  float inv_h, eps;
  int H;
  int attn_S, attn_span, nrb, attn_ctr_base;
  float scale;
  float* gpart;         // split-K partials [unit][NT][128 mpc]
  size_t gpart_unit;    // floats per unit partial
  float* apart;         // attention partials [group][attn_S][64][hd + 4]
  unsigned* ctr;        // this launch's counters [L][ctr_layer], then the abort word
  int ctr_layer;
  int phase_target[kPhases];   // CTAs holding work in each phase
  const uint32_t* tasks;       // [grid][kLoopMaxTasks]: phase << 24 | unit
  const int* ntasks;           // [grid]
  unsigned* status;
  int off_op, off_misc, off_bar, smem_bytes, acc_cols, tmem_cols, mpc_max;
};

__host__ __device__ constexpr int loop_phase_op(int ph) { return ph == PH_QKV ? 0 : ph == PH_O ? 1 : ph == PH_GU ? 2 : 3; }
__device__ __forceinline__ int loop_op_of(int ph) { return loop_phase_op(ph); }

// Bounded wait for a grid-scope counter to reach `target` (acquire).
__device__ __noinline__ bool loop_wait_count(const unsigned* ctr, unsigned target, unsigned* abort_word,
                                             unsigned* status) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (unsigned i = 1;; ++i) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((i & 31u) == 0) {
      if (*reinterpret_cast<volatile unsigned*>(abort_word)) return false;
      if (globaltimer_ns() - t0 > kLoopWaitNs) {
        atomicOr(status, DEV_ERR_TIMEOUT_FLAG);
        atomicExch(abort_word, 1u);
        return false;
      }
    }
  }
}

// Bounded mbarrier wait that also gives up when another CTA raised the abort word.
__device__ __noinline__ bool loop_mbar_wait(uint64_t* bar, uint32_t parity, unsigned* abort_word, unsigned* status,
                                            unsigned err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (unsigned i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (abort_word && *reinterpret_cast<volatile unsigned*>(abort_word)) return false;
      if (globaltimer_ns() - t0 > kLoopWaitNs) {
        atomicOr(status, err);
        if (abort_word) atomicExch(abort_word, 1u);
        return false;
      }
    }
  }
}

template <int HD, int CS>
__global__ void __launch_bounds__(kLoopThreads, 1) loop_kernel(const __grid_constant__ LoopParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int NT = p.NT;
  unsigned* abort_word = p.ctr + (size_t)p.L * p.ctr_layer;

  uint8_t* ring = smem;                                        // [stages][16 KB] weight tiles
  uint8_t* opb = smem + p.off_op;                              // operand slice / attention staging
  float* rpart = reinterpret_cast<float*>(smem + p.off_misc);  // [128]
  float* rstd = rpart + kMathThreads;                          // [NT]
  float* sq = rstd + NT;                                       // [NT][32 mpc_max] (attention: merge weights)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* full = bars;                       // [stages]
  uint64_t* empty = bars + p.stages;           // [stages]
  uint64_t* bfull = bars + 2 * p.stages;       // operand slice landed
  uint64_t* opfree = bfull + 1;                // MMAs reading the operand slice are done
  uint64_t* tfull = opfree + 1;                // [2] accumulator ready
  uint64_t* tempty = tfull + 2;                // [2] accumulator drained
  uint64_t* fin = tempty + 2;                  // all MMAs done (exit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint32_t* s_tasks = tmem_slot + 1;           // [kLoopMaxTasks]
  const int ntask = min(p.ntasks[cta], kLoopMaxTasks);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(bfull, 1);
    mbar_init(opfree, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 1);
    }
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < ntask; i += blockDim.x) s_tasks[i] = p.tasks[(size_t)cta * kLoopMaxTasks + i];
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  // unit geometry of a GEMM task
  struct Unit {
    int op, mg, r, mt0, nmt, kt0, nkt;
  };
  auto unit_of = [&](uint32_t task) {
    Unit u;
    u.op = loop_op_of((int)(task >> 24));
    const LoopOp& o = p.op[u.op];
    const int unit = (int)(task & 0xFFFFFFu);
    u.mg = unit / o.S;
    u.r = unit % o.S;
    u.mt0 = u.mg * o.mpc;
    u.nmt = min(o.mpc, o.Mt - u.mt0);
    u.kt0 = (u.r * o.KBt) / o.S;
    u.nkt = ((u.r + 1) * o.KBt) / o.S - u.kt0;
    return u;
  };
  auto phase_ctr = [&](int l, int ph) { return p.ctr + (size_t)l * p.ctr_layer + ph; };
  auto active = [&](int l, int ph) { return (l > p.l0 || ph >= p.ph0) && (l < p.l1 - 1 || ph < p.ph1); };
  // counter that must be complete before phase `ph` of layer `l` may read its inputs
  auto dep_ok = [&](int l, int ph) -> bool {
    if (l == p.l0 && ph == p.ph0) return true;   // produced by the previous kernel
    const int pl = ph == PH_QKV ? l - 1 : l;
    const int pph = ph == PH_QKV ? PH_D : ph - 1;
    return loop_wait_count(phase_ctr(pl, pph), (unsigned)p.phase_target[pph], abort_word, p.status);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer: weight stream
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;                 // tiles issued so far
      int ps = 0;                 // ring stage of tile `it`
      uint32_t pph = 0;           // round parity of that stage (tile it uses round it / stages)
      bool ok = true;
      for (int l = p.l0; l < p.l1 && ok; ++l) {
        // the prefix K / V^T rows this CTA's attention units will read in layer l: into L2 now,
        // while earlier layers run (16-byte aligned: spans start at multiples of 16 keys)
        for (int ti = 0; ti < ntask; ++ti) {
          const uint32_t task = s_tasks[ti];
          if ((int)(task >> 24) != PH_ATTN || !active(l, PH_ATTN)) continue;
          const int unit = (int)(task & 0xFFFFFFu);
          const int group = unit / p.attn_S, c = unit % p.attn_S;
          const int bk = group / p.nrb;
          const int k0 = c * p.attn_span, k1 = min(p.P, k0 + p.attn_span);
          if (k1 <= k0) continue;
          const size_t cache = (size_t)l * p.cache_layer;
          bulk_prefetch_l2(p.kc + cache + ((size_t)bk * p.Lpad + k0) * HD, (uint32_t)(k1 - k0) * HD * 2);
          const uint32_t vbytes = (uint32_t)(((k1 - k0) * 2 + 15) & ~15);
          for (int dd = 0; dd < HD; ++dd)
            bulk_prefetch_l2(p.vct + cache + ((size_t)bk * HD + dd) * p.Lpad + k0, vbytes);
        }
        for (int ti = 0; ti < ntask && ok; ++ti) {
          const uint32_t task = s_tasks[ti];
          if ((int)(task >> 24) == PH_ATTN || !active(l, (int)(task >> 24))) continue;
          const Unit u = unit_of(task);
          const LoopOp& o = p.op[u.op];
          const uint8_t* src = p.wpack + (size_t)l * p.layer_wbytes + o.woff +
                               ((size_t)u.mt0 * o.KBt + u.kt0) * kTileBytes;
          int li = 0;
          for (int i = 0; i < u.nmt * u.nkt; ++i, ++it) {
            // stage ps is reused once its previous round (parity pph ^ 1) was consumed
            if (it >= p.stages && !mbar_try_wait(&empty[ps], pph ^ 1u) &&
                !(ok = loop_mbar_wait(&empty[ps], pph ^ 1u, abort_word, p.status, DEV_ERR_TIMEOUT_TMA)))
              break;
            mbar_arrive_expect_tx(&full[ps], kTileBytes);
            bulk_g2s(ring + (size_t)ps * kTileBytes, src, kTileBytes, &full[ps], pol);
            src += kTileBytes;
            if (++li == u.nkt) {   // next m-tile of the unit: skip the k-tiles of the other splits
              li = 0;
              src += (size_t)(o.KBt - u.nkt) * kTileBytes;
            }
            if (++ps == p.stages) {
              ps = 0;
              pph ^= 1u;
            }
          }
        }
      }
      // drain: every copy this thread issued has landed before the CTA may exit
      for (int k = max(0, it - p.stages); k < it; ++k)
        loop_mbar_wait(&full[k % p.stages], (k / p.stages) & 1, nullptr, p.status, DEV_ERR_TIMEOUT_TMA);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 2 * NT);   // hi and lo token rows in one MMA
      // descriptors of ring stage 0 and of the operand's first k-block; 16 bytes = one unit of
      // the start-address field (shared addresses stay below 256 KB: no carry out of it)
      const uint64_t a0 = sw128_desc(smem_u32(ring)), b0 = sw128_desc(smem_u32(opb));
      const uint32_t bstride = (uint32_t)NT * 128u;         // bytes of one hi or lo tile
      int it = 0, tcount = 0, opcount = 0, waited = -1;
      int rs = 0;                                           // ring stage of tile `it`
      uint32_t rph = 0;                                     // and its phase parity
      bool ok = true;
      for (int l = p.l0; l < p.l1 && ok; ++l) {
        for (int ti = 0; ti < ntask && ok; ++ti) {
          const uint32_t task = s_tasks[ti];
          const int ph = (int)(task >> 24);
          if (ph == PH_ATTN || !active(l, ph)) continue;
          const Unit u = unit_of(task);
          const LoopOp& o = p.op[u.op];
          if (waited != l * kPhases + ph) {
            if (!(ok = dep_ok(l, ph))) break;
            waited = l * kPhases + ph;
            fence_proxy_async_global();
          }
          // operand slice: the previous unit's MMAs must be done with the buffer
          if (opcount > 0 &&
              !(ok = loop_mbar_wait(opfree, (opcount - 1) & 1, abort_word, p.status, DEV_ERR_TIMEOUT_MMA)))
            break;
          const __nv_bfloat16* act = u.op == 0 ? p.act_x : u.op == 1 ? p.act_o : u.op == 2 ? p.act_x : p.act_m;
          const int kb0 = u.kt0, kb1 = min(u.kt0 + u.nkt, o.KB);
          const uint32_t bytes = (uint32_t)(kb1 - kb0) * 2u * bstride;
          mbar_arrive_expect_tx(bfull, bytes);
          bulk_g2s(opb, act + (size_t)kb0 * 2 * NT * 64, bytes, bfull, policy_evict_last());
          ok = loop_mbar_wait(bfull, opcount & 1, nullptr, p.status, DEV_ERR_TIMEOUT_TMA);   // never left in flight
          ++opcount;
          if (!ok) break;
          const int buf = tcount & 1;
          if (tcount >= 2 &&
              !(ok = loop_mbar_wait(&tempty[buf], ((tcount >> 1) - 1) & 1, abort_word, p.status, DEV_ERR_TIMEOUT_MMA)))
            break;
          tc_fence_after();
          // one thread issues every MMA of the CTA: keep the per-tile work to a ring-stage step
          // (no divisions) and the wait's fast path inline
          uint32_t d_tmem = tmem_d + (uint32_t)(buf * p.acc_cols);
          int li = 0;
          for (int i = 0; i < u.nmt * u.nkt; ++i, ++it) {
            // the mbarrier orders the bulk-copied tile before the MMA reads it (both async proxy)
            if (!mbar_try_wait(&full[rs], rph) &&
                !(ok = loop_mbar_wait(&full[rs], rph, abort_word, p.status, DEV_ERR_TIMEOUT_TMA)))
              break;
            const uint64_t ad = a0 + (uint64_t)((uint32_t)rs * (kTileBytes >> 4));
            const uint64_t bd = b0 + (uint64_t)((uint32_t)li * 2u * (bstride >> 4));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (li | kk) != 0);
            mma_commit(&empty[rs]);
            if (++rs == p.stages) {
              rs = 0;
              rph ^= 1u;
            }
            if (++li == u.nkt) {
              li = 0;
              d_tmem += (uint32_t)(2 * NT);
            }
          }
          if (!ok) break;
          mma_commit(&tfull[buf]);
          mma_commit(opfree);
          ++tcount;
        }
      }
      mma_commit(fin);
      loop_mbar_wait(fin, 0, nullptr, p.status, DEV_ERR_TIMEOUT_MMA);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    const int mtid = threadIdx.x - 64;   // 0..127
    const int quarter = warp & 3;         // TMEM lanes this warp may access
    const int L_all = p.P + p.Ts;
    const int rep = p.nq / p.nkv;
    int tcount = 0;
    bool ok = true;
    auto bar_ok = [&](bool mine) -> bool {   // make thread 0's verdict the warps' verdict
      if (mtid == 0) rpart[0] = mine ? 1.f : 0.f;
      math_bar();
      const bool v = rpart[0] != 0.f;
      math_bar();
      return v;
    };
    // publish this CTA's global writes: one barrier, then one release (device scope) by thread 0
    auto publish = [&](unsigned* ctr) {
      math_bar();
      if (mtid == 0) {
        fence_proxy_async_global();   // consumers may read with bulk copies
        red_release_gpu_add(ctr, 1u);
      }
    };
    for (int l = p.l0; l < p.l1 && ok; ++l) {
      const float* modl = p.mod + (size_t)l * 6 * p.H;
      const size_t cache = (size_t)l * p.cache_layer;
      unsigned* lctr = p.ctr + (size_t)l * p.ctr_layer;
      for (int ph = 0; ph < kPhases && ok; ++ph) {
        int first = -1, count = 0;
        for (int ti = 0; ti < ntask; ++ti)
          if ((int)(s_tasks[ti] >> 24) == ph) {
            if (first < 0) first = ti;
            ++count;
          }
        if (count == 0 || !active(l, ph)) continue;
        if (ph != PH_ATTN && !(ok = bar_ok(mtid == 0 ? dep_ok(l, ph) : true))) break;

        if (ph == PH_ATTN) {
          constexpr int RST = HD + 4;
          // pass A: partial over this task's key span -> global, count it
          for (int ti = first; ti < first + count; ++ti) {
            const int unit = (int)(s_tasks[ti] & 0xFFFFFFu);
            const int group = unit / p.attn_S, c = unit % p.attn_S;
            const int rb = group % p.nrb, bk = group / p.nrb;   // bk = b * nkv + kvh
            const int kbeg = c * p.attn_span, kend = min(L_all, kbeg + p.attn_span);
            float* dst = p.apart + (size_t)unit * kAttnRows * RST;
            // the prefix part of the first sub-chunk does not depend on this step: its copies are
            // issued before the wait for the QKV phase
            bool dep = true;
            attn_block_partial<HD, CS>(
                opb, p.q + ((size_t)bk * p.Rpad + (size_t)rb * kAttnRows) * HD,
                p.kc + cache + (size_t)bk * p.Lpad * HD, p.vct + cache + (size_t)bk * HD * p.Lpad, p.P, p.Lpad, kbeg,
                kend, p.scale, mtid, [] { math_bar(); },
                [&] {
                  if (ti == first) dep = bar_ok(mtid == 0 ? dep_ok(l, ph) : true);
                },
                [&](int r) { return dst + (size_t)r * RST; });
            if (!(ok = dep)) break;   // (the partial read stale rows; nothing is published)
            publish(lctr + p.attn_ctr_base + group);
          }
          if (!ok) break;
          fence_proxy_async_smem();   // the staging area is reused by bulk copies later
          // pass B: merge the rows this span owns once every span of the block is in
          for (int ti = first; ti < first + count && ok; ++ti) {
            const int unit = (int)(s_tasks[ti] & 0xFFFFFFu);
            const int group = unit / p.attn_S, c = unit % p.attn_S;
            const int rb = group % p.nrb, bk = group / p.nrb;
            const int S = p.attn_S;
            const int rpo = (kAttnRows + S - 1) / S;
            const int rbeg = min(kAttnRows, c * rpo), rend = min(kAttnRows, rbeg + rpo), nr = rend - rbeg;
            if (!(ok = bar_ok(mtid == 0 ? loop_wait_count(lctr + p.attn_ctr_base + group, (unsigned)S, abort_word,
                                                          p.status)
                                        : true)))
              break;
            const float* src0 = p.apart + (size_t)group * S * kAttnRows * RST;
            // step 1: per owned row, the weight of each span: 2^(m_s - max) / sum_s 2^(m_s - max) l_s
            float* wts = sq;   // [nr][S]
            for (int e = mtid; e < nr * S; e += kMathThreads) {
              const int r = e / S, s2 = e % S;
              const float2 ml = __ldcg(reinterpret_cast<const float2*>(src0 + ((size_t)s2 * kAttnRows + rbeg + r) * RST + HD));
              wts[e] = ml.x;
              wts[nr * S + e] = ml.y;
            }
            math_bar();
            for (int r = mtid; r < nr; r += kMathThreads) {
              float mx = -INFINITY;
              for (int s2 = 0; s2 < S; ++s2) mx = fmaxf(mx, wts[r * S + s2]);
              float den = 0.f;
              for (int s2 = 0; s2 < S; ++s2) {   // rank order: deterministic
                const float w = exp2f(wts[r * S + s2] - mx);
                wts[r * S + s2] = w;
                den = fmaf(w, wts[nr * S + r * S + s2], den);
              }
              const float inv = 1.f / den;
              for (int s2 = 0; s2 < S; ++s2) wts[r * S + s2] *= inv;
            }
            math_bar();
            // step 2: weighted sum of the spans' O rows, 4 dims per item, 8 loads in flight
            const int row_base = rb * kAttnRows, R = rep * p.Ts;
            for (int e = mtid; e < nr * (HD / 4); e += kMathThreads) {
              const int r = e / (HD / 4), d = (e % (HD / 4)) * 4;
              const int row = row_base + rbeg + r;
              if (row >= R) continue;
              float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int s0 = 0; s0 < S; s0 += 8) {
                float4 v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  if (s0 + k < S)
                    v[k] = __ldcg(reinterpret_cast<const float4*>(src0 + ((size_t)(s0 + k) * kAttnRows + rbeg + r) * RST + d));
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  if (s0 + k < S) {
                    const float w = wts[r * S + s0 + k];
                    acc.x = fmaf(w, v[k].x, acc.x);
                    acc.y = fmaf(w, v[k].y, acc.y);
                    acc.z = fmaf(w, v[k].z, acc.z);
                    acc.w = fmaf(w, v[k].w, acc.w);
                  }
              }
              const int head = (bk % p.nkv) * rep + row / p.Ts, tok = (bk / p.nkv) * p.Ts + row % p.Ts;
              __nv_bfloat16 hi[4], lo[4];
              split_bf16(acc.x, hi[0], lo[0]);
              split_bf16(acc.y, hi[1], lo[1]);
              split_bf16(acc.z, hi[2], lo[2]);
              split_bf16(acc.w, hi[3], lo[3]);
              __nv_bfloat16* base = p.act_o + operand_offset(tok, head * HD + d, NT, p.op[1].KB);
              *reinterpret_cast<uint2*>(base) = *reinterpret_cast<const uint2*>(hi);
              *reinterpret_cast<uint2*>(base + (size_t)NT * 64) = *reinterpret_cast<const uint2*>(lo);
            }
            math_bar();   // wts is reused by the next task
          }
        } else {
          const int oi = loop_op_of(ph);
          const LoopOp& o = p.op[oi];
          const bool norm = ph == PH_QKV || ph == PH_GU;
          if (norm) {
            // rstd per token row from the partial sums of squares: G threads per row, 8 loads in
            // flight per thread, fixed summation order (deterministic); overlaps the MMAs
            const int parts = ph == PH_QKV ? (l == p.l0 ? p.ss_parts_first : p.op[3].parts_out) : p.op[1].parts_out;
            const int rows = min(NT, p.Ntok);
            const int G = max(1, kMathThreads / rows);
            const int row = mtid / G, g = mtid % G;
            float a[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) a[k] = 0.f;
            if (row < rows) {
              int q = g;
              for (; q + 7 * G < parts; q += 8 * G) {
                float v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = __ldcg(p.ss + (size_t)(q + k * G) * p.Ntok + row);
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] += v[k];
              }
#pragma unroll
              for (int k = 0; k < 8; ++k)   // the last fewer-than-8 parts
                if (q + k * G < parts) a[k] += __ldcg(p.ss + (size_t)(q + k * G) * p.Ntok + row);
            }
            rpart[mtid] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
            math_bar();
            for (int r = mtid; r < NT; r += kMathThreads) {
              float s2 = 0.f;
              if (r < rows)
                for (int gg = 0; gg < G; ++gg) s2 += rpart[r * G + gg];
              rstd[r] = rsqrtf(s2 * p.inv_h + p.eps);
            }
            math_bar();
          }
          // pass A: accumulators -> split partials in global memory ([unit][NT][rows], fp32)
          for (int ti = first; ti < first + count && ok; ++ti) {
            const Unit u = unit_of(s_tasks[ti]);
            const int buf = tcount & 1;
            // one thread waits, all follow its verdict (a split verdict would strand a named barrier)
            if (!(ok = bar_ok(mtid == 0 ? loop_mbar_wait(&tfull[buf], (tcount >> 1) & 1, abort_word, p.status,
                                                         DEV_ERR_TIMEOUT_MMA)
                                        : true)))
              break;
            tc_fence_after();
            float* dst = p.gpart + (size_t)(u.mg * o.S + u.r) * p.gpart_unit;
            const int rows = u.nmt * 128;
            const int ncols = min(NT, p.Ntok);   // token columns past Ntok are padding: not stored
            for (int j = 0; j < u.nmt; ++j) {
              const int row = j * 128 + quarter * 32 + lane;
              for (int c0 = 0; c0 < ncols; c0 += 16) {
                float vh[16], vl[16];
                const uint32_t ta = tmem_d + (uint32_t)(buf * p.acc_cols) + ((uint32_t)(quarter * 32) << 16) +
                                    (uint32_t)(j * 2 * NT + c0);
                tmem_ld16(ta, vh);
                tmem_ld16(ta + (uint32_t)NT, vl);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c)
                  if (c0 + c < ncols) __stcg(dst + (size_t)(c0 + c) * rows + row, vh[c] + vl[c]);
              }
            }
            tc_fence_before();
            math_bar();
            if (mtid == 0) {
              mbar_arrive(&tempty[buf]);
              if (o.S > 1) red_release_gpu_add(lctr + o.ctr_base + u.mg, 1u);
            }
            ++tcount;
          }
          // pass B: reduce the rows this split owns, fused epilogue.  A work item is one token
          // column and 4 consecutive packed rows (2 RoPE pairs, 2 gate/up pairs, or 4 rows).
          // Everything an item reads that does not depend on the other splits (epilogue vectors,
          // residual, RoPE factors) is loaded together with its partials: one round trip.
          // Per-output-row vectors of this (step, layer): W.shift of the norm ops, gate and the
          // next op's modulation scale of the residual ops.
          const float* vcs = ph == PH_QKV ? p.cq + (size_t)l * p.cq_stride
                           : ph == PH_GU  ? p.cg + (size_t)l * p.cg_stride : nullptr;
          const float* vga = ph == PH_O ? modl + 2 * p.H : ph == PH_D ? modl + 5 * p.H : nullptr;
          const float* vsn = ph == PH_O ? modl + 4 * p.H : (ph == PH_D && l + 1 < p.L) ? modl + 7 * p.H : nullptr;
          for (int ti = first; ti < first + count && ok; ++ti) {
            const Unit u = unit_of(s_tasks[ti]);
            const int S = o.S;
            const int rows = u.nmt * 128, n4 = u.nmt * 32, U = n4 * NT;
            for (int i = mtid; i < NT * n4; i += kMathThreads) sq[i] = 0.f;
            bool mine = true;
            if (S > 1 && mtid == 0)
              mine = loop_wait_count(lctr + o.ctr_base + u.mg, (unsigned)S, abort_word, p.status);
            if (!(ok = bar_ok(mine))) break;
            const int ub0 = (u.r * U) / S, ub1 = ((u.r + 1) * U) / S;
            const float* src0 = p.gpart + (size_t)(u.mg * S) * p.gpart_unit;
            for (int un = ub0 + mtid; un < ub1; un += kMathThreads) {
              const int col = un / n4, quad = un % n4;   // consecutive threads: consecutive rows
              const int t = col;
              const int o0 = u.mt0 * 128 + quad * 4;     // first of 4 packed output rows
              if (t >= p.Ntok || o0 >= o.O) continue;
              const int nv = min(4, o.O - o0);
              float cs[4], gt[4], sc[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                cs[q] = (vcs && q < nv) ? __ldg(vcs + o0 + q) : 0.f;
                gt[q] = (vga && q < nv) ? __ldg(vga + o0 + q) : 0.f;
                sc[q] = (vsn && q < nv) ? __ldg(vsn + o0 + q) : 0.f;
              }
              float* hp = p.h + (size_t)t * o.O + o0;
              float4 hv = make_float4(0.f, 0.f, 0.f, 0.f);
              if ((ph == PH_O || ph == PH_D) && nv == 4) hv = __ldcg(reinterpret_cast<const float4*>(hp));
              const int qd = p.nq * HD, kd = p.nkv * HD, half = HD >> 1;
              const int jt = t % p.Ts;
              float4 rp = make_float4(0.f, 0.f, 0.f, 0.f);
              if (ph == PH_QKV && o0 < qd + kd) {
                const int local = o0 < qd ? o0 : o0 - qd;
                rp = __ldg(reinterpret_cast<const float4*>(p.rope + 2 * ((size_t)jt * half + ((local % HD) >> 1))));
              }
              float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
              const float* sp = src0 + (size_t)col * rows + quad * 4;
              for (int s0 = 0; s0 < S; s0 += 8) {   // 8 loads in flight, summed in rank order
                float4 v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  if (s0 + k < S) v[k] = __ldcg(reinterpret_cast<const float4*>(sp + (size_t)(s0 + k) * p.gpart_unit));
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  if (s0 + k < S) {
                    y.x += v[k].x;
                    y.y += v[k].y;
                    y.z += v[k].z;
                    y.w += v[k].w;
                  }
              }
              if (norm) {
                const float rs = rstd[col];
                y.x = fmaf(rs, y.x, cs[0]);
                y.y = fmaf(rs, y.y, cs[1]);
                y.z = fmaf(rs, y.z, cs[2]);
                y.w = fmaf(rs, y.w, cs[3]);
              }
              if (ph == PH_O || ph == PH_D) {
                float hn[4];
                if (nv == 4) {
                  hn[0] = fmaf(gt[0], y.x, hv.x);
                  hn[1] = fmaf(gt[1], y.y, hv.y);
                  hn[2] = fmaf(gt[2], y.z, hv.z);
                  hn[3] = fmaf(gt[3], y.w, hv.w);
                  __stcg(reinterpret_cast<float4*>(hp), make_float4(hn[0], hn[1], hn[2], hn[3]));
                } else {   // ragged end of the hidden rows
                  const float yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                  for (int q = 0; q < 4; ++q) hn[q] = q < nv ? fmaf(gt[q], yy[q], __ldcg(hp + q)) : 0.f;
                  for (int q = 0; q < nv; ++q) __stcg(hp + q, hn[q]);
                }
                sq[col * n4 + quad] = ((hn[0] * hn[0] + hn[1] * hn[1]) + hn[2] * hn[2]) + hn[3] * hn[3];
                if (ph == PH_O || l + 1 < p.L) {   // next GEMM's operand h (1 + scale); zero past the row end
                  __nv_bfloat16 hi[4], lo[4];
#pragma unroll
                  for (int q = 0; q < 4; ++q) split_bf16(hn[q] * (1.f + sc[q]), hi[q], lo[q]);
                  const int KBn = ph == PH_O ? p.op[2].KB : p.op[0].KB;
                  __nv_bfloat16* bn = p.act_x + operand_offset(t, o0, NT, KBn);
                  *reinterpret_cast<uint2*>(bn) = *reinterpret_cast<const uint2*>(hi);
                  *reinterpret_cast<uint2*>(bn + (size_t)NT * 64) = *reinterpret_cast<const uint2*>(lo);
                }
              } else if (ph == PH_GU) {
                // rows (2j, 2j+1) = (gate_j, up_j): two SwiGLU outputs
                __nv_bfloat16 hi[2], lo[2];
                split_bf16(y.x / (1.f + __expf(-y.x)) * y.y, hi[0], lo[0]);
                split_bf16(y.z / (1.f + __expf(-y.z)) * y.w, hi[1], lo[1]);
                __nv_bfloat16* mb = p.act_m + operand_offset(t, o0 >> 1, NT, p.op[3].KB);
                *reinterpret_cast<uint32_t*>(mb) = *reinterpret_cast<const uint32_t*>(hi);
                *reinterpret_cast<uint32_t*>(mb + (size_t)NT * 64) = *reinterpret_cast<const uint32_t*>(lo);
              } else {   // QKV: RoPE, q and the self rows of the layer's K / V^T caches
                const int b = t / p.Ts;
                if (o0 < qd + kd) {
                  // rotary pairs i0, i0 + 1 of one head: x_i in even rows, x_{i+hd/2} in odd rows
                  const bool isq = o0 < qd;
                  const int local = isq ? o0 : o0 - qd;
                  const int head = local / HD, i0 = (local % HD) >> 1;
                  const __nv_bfloat162 e0 = __floats2bfloat162_rn(y.x * rp.x - y.y * rp.y, y.z * rp.z - y.w * rp.w);
                  const __nv_bfloat162 e1 = __floats2bfloat162_rn(y.y * rp.x + y.x * rp.y, y.w * rp.z + y.z * rp.w);
                  __nv_bfloat16* dst =
                      isq ? p.q + (((size_t)b * p.nkv + head / rep) * p.Rpad + (head % rep) * p.Ts + jt) * HD
                          : p.kc + cache + (((size_t)b * p.nkv + head) * p.Lpad + p.P + jt) * HD;
                  *reinterpret_cast<__nv_bfloat162*>(dst + i0) = e0;
                  *reinterpret_cast<__nv_bfloat162*>(dst + i0 + half) = e1;
                } else {
                  const int local = o0 - qd - kd;
                  const int head = local / HD, d0 = local % HD;
                  __nv_bfloat16* dst = p.vct + cache + (((size_t)b * p.nkv + head) * HD + d0) * p.Lpad + p.P + jt;
                  dst[0] = __float2bfloat16_rn(y.x);
                  dst[(size_t)p.Lpad] = __float2bfloat16_rn(y.y);
                  dst[(size_t)2 * p.Lpad] = __float2bfloat16_rn(y.z);
                  dst[(size_t)3 * p.Lpad] = __float2bfloat16_rn(y.w);
                }
              }
            }
            if (ph == PH_O || ph == PH_D) {
              math_bar();
              for (int col = mtid; col < min(NT, p.Ntok); col += kMathThreads) {
                float acc = 0.f;
                for (int q = 0; q < n4; ++q) acc += sq[col * n4 + q];
                p.ss[(size_t)(u.mg * S + u.r) * p.Ntok + col] = acc;
              }
            }
            math_bar();   // sq / vectors are reused by the next unit
          }
        }
        if (!ok) break;
        publish(phase_ctr(l, ph));   // phase done on this CTA
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, p.tmem_cols);
  }
}

}  // namespace vla
