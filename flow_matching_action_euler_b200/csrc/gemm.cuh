// Skinny weight-streaming GEMM for the action expert's linears, y[t][o] = sum_k W[o][k] x[t][k].
//
// Swap-AB: the weight's output rows are the tcgen05 M side (128 rows per tile) and the few
// tokens (batch x self tokens, padded to a multiple of 32) are the N side, so one M=128 x
// N=NT x K=16 MMA consumes a whole 128-row strip of weights.  At batch 1 the loop is bound by
// the weight stream from HBM ("跨XPU平台表征视觉-语言-动作模型" section 4.2: the action expert is
// memory-bound), so the kernel is organised around keeping that stream full:
//
//  * weights are pre-packed at create time into 16 KB tiles (128 rows x 64 bf16, or 128 rows x
//    128 e4m3) already laid out in the 128-byte swizzle the MMA reads, stored [m-tile][k-block]
//    so every CTA's share is one contiguous range per m-tile, fetched with 1-D bulk copies;
//  * the producer warp issues those copies before `griddepcontrol.wait`, i.e. while the previous
//    kernel of the loop is still running (programmatic dependent launch), on the SMs that kernel
//    leaves free; the ring is as deep as the CTA's share of tiles (up to 8 stages, most of the
//    SM's shared memory), which measured faster than two shallower CTAs per SM;
//  * the activation operand is a pair of bf16 tiles (hi, lo = x - hi) written by the producing
//    kernel in the swizzled layout and fetched with one bulk copy; the two tiles are adjacent, so
//    one MMA with N = 2 NT multiplies both (measured on B200: a 16 KB tile's four M=128 K=16 MMAs
//    take ~350 cycles at N = 64 and ~500 at N = 256, so the lo rows cost little) and the epilogue
//    adds the two column halves: the product is fp32-accurate in the activations while the
//    weights stay exact bf16;
//  * RMSNorm + adaLN modulate ("AI Infra如何优化VLA" section 算子开发) are applied by linearity:
//    W (rms(h) (1 + scale) + shift) = rstd * W (h (1 + scale)) + W shift, so producers write
//    h (1 + scale), this kernel scales by rstd (from partial sums of squares) in the epilogue and
//    adds the input-independent W shift table;
//  * split-K across the CTAs of a thread-block cluster, reduced through distributed shared
//    memory in a fixed order (deterministic, no float atomics);
//  * fused epilogues: RoPE (half-split rotation) writing q and the layer's K / V^T caches, SwiGLU
//    (section 算子融合) writing the down GEMM's operand, and the gated residual add writing h,
//    per-row partial sums of squares and the next GEMM's operand.
//
// Warp roles (192 threads): warp 0 = bulk-copy producer, warp 1 = MMA issuer (and TMEM owner),
// warps 2..5 = math warps (rstd, fp8 -> bf16 conversion, TMEM read-out, epilogue).
#pragma once
#include "ptx.cuh"

namespace vla {

enum EpiKind : int { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

constexpr int kGemmThreads = 192;
constexpr int kMathThreads = 128;
constexpr int kTileBytes = 16384;      // one packed weight tile
constexpr int kConvStages = 2;         // packed-code paths: converted bf16 A stages (KPT x 16 KB each)
constexpr int kMaxMpc = 4;             // m-tiles per CTA

struct GemmParams {
  // ---- A operand (packed weights)
  const uint8_t* w;        // tiles [Mt][KBt][16 KB]
  const float* wscale;     // 8-bit codes: scale per packed row; int4: [packed row][spr] (else nullptr)
  int spr;                 // scales per packed row (int4: one per 128 inputs)
  int Mt;                  // 128-row output tiles
  int mpc;                 // m-tiles per CTA (sharing the activation operand)
  int KBt;                 // weight tiles along K (64 wide for bf16, 128 wide for fp8)
  int K;                   // logical reduction length
  int S;                   // K splits = cluster size along x
  int stages;              // weight-tile ring depth
  // ---- tokens / activation operand
  int Ntok;                // valid token rows
  int NT;                  // token rows per n-tile (multiple of 32, <= 256)
  int KB;                  // 64-wide k-blocks of the operand = ceil(K / 64)
  const __nv_bfloat16* act;  // operand tiles [Nt][KB][2 (hi, lo)][NT][64]
  // ---- normalised input (QKV, gate/up): y = rstd * acc + cshift
  const float* ss;           // partial sums of squares of the residual [ss_parts][Ntok]
  int ss_parts;
  const float* cshift;       // [O] = W . shift for this (step, layer)
  float inv_h, eps;          // 1 / H, RMSNorm epsilon
  // ---- epilogue
  int O;                     // packed output rows
  float* h;                  // RESID: residual [Ntok][O] updated in place
  const float* gate;         // RESID: [O]
  float* ss_out;             // RESID: [Mt / mpc * S][Ntok]
  __nv_bfloat16* b_next;     // RESID: next GEMM's operand tiles [Nt][KBn][2][NT][64] (or nullptr)
  const float* sc_next;      // RESID: next GEMM's modulation scale [O]
  int KBn;
  __nv_bfloat16* m_out;      // SWIGLU: down-GEMM operand tiles [Nt][KBm][2][NT][64]
  int KBm;
  __nv_bfloat16* q_out;      // QKV: q [B][nkv][Rpad][hd] bf16, row = head_in_group * Ts + token
  int Rpad;                  // QKV: padded q rows per kv head (64-row attention blocks)
  __nv_bfloat16* kc;         // QKV: layer K cache [B][nkv][Lpad][hd]
  __nv_bfloat16* vct;        // QKV: layer V^T cache [B][nkv][hd][Lpad]
  const float* rope;         // QKV: [Ts][hd/2][2] (cos, sin) for positions P + j
  int nq, nkv, hd, Ts, P, Lpad;
  const uint8_t* pf_next;     // weights of the next GEMM of the loop: prefetched into L2 (or nullptr)
  size_t pf_bytes;
  unsigned* status;
  // ---- shared-memory layout (bytes from the 1024-aligned base)
  int off_b, off_conv, off_bar, off_misc, off_vec, smem_bytes;
};

__device__ __forceinline__ void math_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// hi/lo bf16 pair of one fp32 value (x = hi + lo to ~2^-16 relative)
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// WQ: weight format, 0 bf16 tiles, 1 e4m3 codes, 2 int8 codes (8-bit formats carry one fp32 scale
// per output row, applied in the epilogue, and are widened to bf16 tiles on chip before the MMA)
template <int EPI, int WQ, bool NORM>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_stream_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool FP8 = WQ != 0;   // 8-bit packed weights (e4m3 or int8)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S;
  const int r = blockIdx.x;          // rank inside the cluster (cluster dims = (S,1,1), grid.x = S)
  const int mg = blockIdx.y, nt = blockIdx.z;
  const int mpc = p.mpc;
  const int mt0 = mg * mpc;
  const int nmt = min(mpc, p.Mt - mt0);
  const int kt0 = (r * p.KBt) / S, kt1 = ((r + 1) * p.KBt) / S, nkt = kt1 - kt0;
  constexpr int KPT = WQ == 3 ? 4 : FP8 ? 2 : 1;   // 64-wide k-blocks per weight tile
  constexpr bool ROW_SCALE = WQ == 1 || WQ == 2;     // scale applied in the epilogue
  const int kb0 = kt0 * KPT;
  const int kb1 = min(kt1 * KPT, p.KB);
  const int NT = p.NT;
  const int ntiles = nmt * nkt;      // weight tiles this CTA streams (m-tile major)
  // split-K epilogue ownership: the nmt * 64 row pairs form octets of 8 pairs; rank q owns octets
  // [q n8 / S, (q + 1) n8 / S).  An epilogue unit is (token column, owned octet).
  const int npairs_all = nmt * 64, n8 = npairs_all / 8;
  const int my_o0 = (r * n8) / S, my_o1 = ((r + 1) * n8) / S;
  const int my_units = (my_o1 - my_o0) * NT;
  float4 pre[4];                     // prefetched residual (RESID) or RoPE (QKV) of the first unit
#pragma unroll
  for (int q = 0; q < 4; ++q) pre[q] = make_float4(0.f, 0.f, 0.f, 0.f);

  uint8_t* sA = smem;                                     // weight ring (and later the reduction buffer)
  uint8_t* sB = smem + p.off_b;                           // operand tiles (hi, lo) of this CTA's k-range
  uint8_t* sC = smem + p.off_conv;                        // fp8: converted bf16 A stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* full = bars;                                  // [stages]
  uint64_t* empty = bars + p.stages;                      // [stages]
  uint64_t* bfull = bars + 2 * p.stages;
  uint64_t* done = bfull + 1;
  uint64_t* cfull = done + 1;                             // [kConvStages]
  uint64_t* cempty = cfull + kConvStages;                 // [kConvStages]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + kConvStages);
  float* rpart = reinterpret_cast<float*>(smem + p.off_misc);   // [128] partial sums of squares
  float* rstd = rpart + kMathThreads;                           // [NT], then [NT][npairs] row sums
  // per-output-row epilogue vectors of this CTA's rows: W.shift | gate | next scale | fp8 scale
  float* v_cshift = reinterpret_cast<float*>(smem + p.off_vec);
  float* v_gate = v_cshift + mpc * 128;
  float* v_scn = v_gate + mpc * 128;
  float* v_wsc = v_scn + mpc * 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], FP8 ? kMathThreads : 1);
    }
    mbar_init(bfull, 1);
    mbar_init(done, 1);
    for (int i = 0; i < kConvStages; ++i) {
      mbar_init(&cfull[i], kMathThreads);
      mbar_init(&cempty[i], 1);
    }
    fence_mbar_init();
  }
  const bool stacked = 2 * NT <= 256;     // hi and lo rows in one MMA (else two MMAs, N = NT)
  const int acc_cols = mpc * 2 * NT;      // per m-tile: hi columns [0,NT), lo columns [NT,2NT)
  const int tmem_cols = acc_cols <= 32 ? 32 : acc_cols <= 64 ? 64 : acc_cols <= 128 ? 128 : acc_cols <= 256 ? 256 : 512;
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();

  auto tile_src = [&](int i) {   // i-th weight tile of this CTA: m-tile mt0 + i / nkt, k-tile kt0 + i % nkt
    return p.w + ((size_t)(mt0 + i / nkt) * p.KBt + kt0 + i % nkt) * kTileBytes;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer: weight stream
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int prefill = min(ntiles, p.stages);
      // the first ring's worth of weights does not depend on the previous kernel
      for (int i = 0; i < prefill; ++i) {
        mbar_arrive_expect_tx(&full[i], kTileBytes);
        bulk_g2s(sA + (size_t)i * kTileBytes, tile_src(i), kTileBytes, &full[i], pol);
      }
      // the rest of this CTA's weights, then this CTA's slice of the next GEMM's weights, go to
      // L2 now so HBM keeps streaming while the loop waits on the previous kernel
      for (int i = prefill; i < ntiles;) {
        const int j = i / nkt;
        const int n = min(ntiles, (j + 1) * nkt) - i;   // contiguous run inside one m-tile
        bulk_prefetch_l2(tile_src(i), (uint32_t)n * kTileBytes);
        i += n;
      }
      if (p.pf_next) {
        const size_t nctas = (size_t)gridDim.x * gridDim.y * gridDim.z;
        const size_t cta = blockIdx.x + (size_t)gridDim.x * (blockIdx.y + (size_t)gridDim.y * blockIdx.z);
        const size_t chunk = ((p.pf_bytes + nctas - 1) / nctas + 4095) & ~size_t(4095);
        const size_t b0 = cta * chunk;
        if (b0 < p.pf_bytes) bulk_prefetch_l2(p.pf_next + b0, (uint32_t)min(chunk, p.pf_bytes - b0));
      }
      // activation tiles are produced by the previous kernel: only after its completion
      pdl_wait();
      const uint32_t bytes = (uint32_t)(kb1 - kb0) * 2u * NT * 128u;
      mbar_arrive_expect_tx(bfull, bytes);
      bulk_g2s(sB, p.act + ((size_t)nt * p.KB + kb0) * 2 * NT * 64, bytes, bfull, policy_evict_last());
      if (prefill < ntiles) {
        // tile i reuses stage i % stages once round i / stages - 1 of that stage was consumed
        int s = 0, li = prefill % nkt;      // prefill == stages here, so tile `prefill` opens stage 0
        uint32_t ph = 0;
        const uint8_t* src = tile_src(prefill);
        for (int i = prefill; i < ntiles; ++i) {
          if (!mbar_wait(&empty[s], ph, p.status, DEV_ERR_TIMEOUT_TMA)) break;
          mbar_arrive_expect_tx(&full[s], kTileBytes);
          bulk_g2s(sA + (size_t)s * kTileBytes, src, kTileBytes, &full[s], pol);
          src += kTileBytes;
          if (++li == nkt) {                // next m-tile: skip the k-tiles other ranks stream
            li = 0;
            src += (size_t)(p.KBt - nkt) * kTileBytes;
          }
          if (++s == p.stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, stacked ? 2 * NT : NT);
      bool ok = mbar_wait(bfull, 0, p.status, DEV_ERR_TIMEOUT_TMA);
      const uint32_t bstride = (uint32_t)NT * 128u;   // bytes of one hi or lo tile
      // descriptors of the first A stage and of the first operand k-block; a step of 16 bytes is
      // one unit of the descriptor's start-address field (shared addresses stay below 256 KB, so
      // adding offsets never carries out of that field).  This issue loop runs in one thread and
      // sits on the kernel's critical path: no divisions, no descriptor rebuilds per tile.
      const uint64_t a0 = sw128_desc(smem_u32(FP8 ? sC : sA)), b0 = sw128_desc(smem_u32(sB));
      const uint64_t lo_off = bstride >> 4;           // hi tile -> lo tile
      // one (hi ++ lo) product per K step when stacked, else hi into cols [0,NT), lo into [NT,2NT)
      auto mma_k = [&](uint32_t d_tmem, uint64_t ad, uint64_t bd, uint32_t acc) {
        mma_bf16(d_tmem, ad, bd, idesc, acc);
        if (!stacked) mma_bf16(d_tmem + (uint32_t)NT, ad, bd + lo_off, idesc, acc);
      };
      int s = 0, li = 0;                              // ring / conversion stage, local k-tile
      uint32_t ph = 0;                                // its phase parity
      uint32_t d_tmem = tmem_d;                       // accumulator of the current m-tile
      for (int i = 0; i < ntiles && ok; ++i) {
        if (!FP8) {
          ok = mbar_wait(&full[s], ph, p.status, DEV_ERR_TIMEOUT_TMA);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = a0 + (uint64_t)((uint32_t)s * (kTileBytes >> 4));
          const uint64_t bd = b0 + (uint64_t)((uint32_t)li * 2u * lo_off);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_k(d_tmem, ad + 2 * kk, bd + 2 * kk, (li | kk) != 0);
          mma_commit(&empty[s]);
          if (++s == p.stages) {
            s = 0;
            ph ^= 1u;
          }
        } else {
          ok = mbar_wait(&cfull[s], ph, p.status, DEV_ERR_TIMEOUT_CONV);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < KPT; ++half) {
            const int lkb = li * KPT + half;                    // local 64-wide k-block
            if (kb0 + lkb >= kb1) break;                        // ragged K tail
            const uint64_t ad = a0 + (uint64_t)((uint32_t)(s * KPT + half) * (kTileBytes >> 4));
            const uint64_t bd = b0 + (uint64_t)((uint32_t)lkb * 2u * lo_off);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_k(d_tmem, ad + 2 * kk, bd + 2 * kk, (lkb | kk) != 0);
          }
          mma_commit(&cempty[s]);
          if (++s == kConvStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (++li == nkt) {
          li = 0;
          d_tmem += (uint32_t)(2 * NT);
        }
      }
      mma_commit(done);
      // the epilogue warps learn that the accumulators are complete from the barrier below (one
      // polling thread instead of four polling warps)
      mbar_wait(done, 0, p.status, DEV_ERR_TIMEOUT_MMA);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    const int mtid = threadIdx.x - 64;   // 0..127
    int conv_done = 0;
    auto convert_one = [&](int i) -> bool {
      // 8-bit tile (128 rows x 128 B, swizzled by 16 B chunks) -> two bf16 SW128 tiles;
      // int4 tile (128 rows x 256 codes) -> four, each code times its group's scale
      const int s = i % p.stages, c = i % kConvStages;
      float gsc[8];
      if constexpr (WQ == 3) {   // the group scales of this thread's 8 chunks, before any wait
        const int j = i / nkt, kt = kt0 + i % nkt;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int idx = mtid + jj * kMathThreads, row = idx >> 3, ch = idx & 7;
          // chunks past K hold zero codes; their group index is clamped to stay inside the row
          const int g = min(kt * 2 + (ch >> 2), p.spr - 1);
          gsc[jj] = __ldg(p.wscale + (size_t)((mt0 + j) * 128 + row) * p.spr + g);
        }
      }
      if (!mbar_wait(&full[s], (i / p.stages) & 1, p.status, DEV_ERR_TIMEOUT_TMA)) return false;
      if (i >= kConvStages && !mbar_wait(&cempty[c], ((i / kConvStages) - 1) & 1, p.status, DEV_ERR_TIMEOUT_CONV))
        return false;
      const uint8_t* src = sA + (size_t)s * kTileBytes;
      uint8_t* dst = sC + (size_t)c * KPT * kTileBytes;
      if constexpr (WQ == 3) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int idx = mtid + jj * kMathThreads;   // 0..1023: (row, 32-code chunk)
          const int row = idx >> 3, ch = idx & 7;
          const uint4 raw = *reinterpret_cast<const uint4*>(src + sw128_chunk_byte(row, ch));
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
          const float sc = gsc[jj];
          uint8_t* t = dst + (ch >> 1) * kTileBytes;   // which 64-wide bf16 tile
          const int bch = (ch & 1) * 4;                 // its first 8-element chunk
#pragma unroll
          for (int q = 0; q < 4; ++q) {                 // codes 8q .. 8q+7 -> one bf16 chunk
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c0 = (int)((w4[q] >> (8 * e)) & 0xFu), c1 = (int)((w4[q] >> (8 * e + 4)) & 0xFu);
              __nv_bfloat162 b2 = __floats2bfloat162_rn((float)((c0 ^ 8) - 8) * sc, (float)((c1 ^ 8) - 8) * sc);
              o[e] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(t + sw128_chunk_byte(row, bch + q)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      } else {
#pragma unroll 4
      for (int jj = 0; jj < 8; ++jj) {
        const int idx = mtid + jj * kMathThreads;   // 0..1023: (row, fp8 chunk)
        const int row = idx >> 3, ch = idx & 7;
        const uint4 raw = *reinterpret_cast<const uint4*>(src + sw128_chunk_byte(row, ch));
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          o[2 * q] = q8x2_to_bf16x2<WQ>((uint16_t)(w4[q] & 0xFFFFu));
          o[2 * q + 1] = q8x2_to_bf16x2<WQ>((uint16_t)(w4[q] >> 16));
        }
        const int half = ch >> 2;                // which 64-wide bf16 tile
        const int bch = (ch & 3) * 2;            // first bf16 chunk (8 elements) inside it
        uint8_t* t = dst + half * kTileBytes;
        *reinterpret_cast<uint4*>(t + sw128_chunk_byte(row, bch)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(t + sw128_chunk_byte(row, bch + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      }
      fence_proxy_async_smem();
      mbar_arrive(&cfull[c]);
      mbar_arrive(&empty[s]);
      return true;
    };
    // the epilogue's per-row vectors are input-independent: stage them before waiting
    for (int i = mtid; i < nmt * 128; i += kMathThreads) {
      const int o = mt0 * 128 + i;
      const bool in = o < p.O;
      if (NORM) v_cshift[i] = in ? __ldg(p.cshift + o) : 0.f;
      if (EPI == EPI_RESID) {
        v_gate[i] = in ? __ldg(p.gate + o) : 0.f;
        v_scn[i] = (in && p.sc_next) ? __ldg(p.sc_next + o) : 0.f;
      }
      if (ROW_SCALE) v_wsc[i] = in ? __ldg(p.wscale + o) : 0.f;
    }
    bool ok = true;
    if (FP8) {
      // weights do not depend on the previous kernel: convert the first stages before waiting
      const int pre = min(ntiles, kConvStages);
      for (; conv_done < pre && ok; ++conv_done) ok = convert_one(conv_done);
    }
    pdl_wait();
    if (NORM) {
      // rstd per token row from the producers' partial sums of squares: G threads per row each
      // take every G-th part, then the G partials are added in a fixed order (deterministic)
      const int G = NT >= kMathThreads ? 1 : kMathThreads / NT;
      for (int base = 0; base < NT; base += kMathThreads / G) {
        const int row = base + mtid / G, g = mtid % G;
        const int t = nt * NT + row;
        float acc = 0.f;
        if (row < NT && t < p.Ntok) {
          int q = g;
          for (; q + 3 * G < p.ss_parts; q += 4 * G) {
            const float a0 = __ldcg(p.ss + (size_t)q * p.Ntok + t);
            const float a1 = __ldcg(p.ss + (size_t)(q + G) * p.Ntok + t);
            const float a2 = __ldcg(p.ss + (size_t)(q + 2 * G) * p.Ntok + t);
            const float a3 = __ldcg(p.ss + (size_t)(q + 3 * G) * p.Ntok + t);
            acc += a0;
            acc += a1;
            acc += a2;
            acc += a3;
          }
          for (; q < p.ss_parts; q += G) acc += __ldcg(p.ss + (size_t)q * p.Ntok + t);
        }
        rpart[mtid] = acc;
        math_bar();
        if (mtid < kMathThreads / G) {
          const int rr = base + mtid;
          float s2 = 0.f;
          for (int gg = 0; gg < G; ++gg) s2 += rpart[mtid * G + gg];
          if (rr < NT) rstd[rr] = rsqrtf(s2 * p.inv_h + p.eps);
        }
        math_bar();
      }
    }
    // epilogue inputs that the previous kernel produced (residual rows) or that are static
    // (RoPE factors): fetch them for this thread's first epilogue unit while the MMAs run
    if (mtid < my_units) {
      const int col = mtid % NT, oc = mtid / NT;
      const int pr0 = (my_o0 + oc) * 8, j = pr0 >> 6;
      const int t = nt * NT + col;
      const int o0 = (mt0 + j) * 128 + 2 * (pr0 & 63);
      if (EPI == EPI_RESID && t < p.Ntok && o0 + 16 <= p.O) {
        const float4* hp = reinterpret_cast<const float4*>(p.h + (size_t)t * p.O + o0);
#pragma unroll
        for (int q = 0; q < 4; ++q) pre[q] = __ldcg(hp + q);
      }
      if (EPI == EPI_QKV && t < p.Ntok && o0 < p.nq * p.hd + p.nkv * p.hd) {
        const int local = o0 < p.nq * p.hd ? o0 : o0 - p.nq * p.hd;
        const int i0 = (local % p.hd) >> 1, half = p.hd >> 1, jt = t % p.Ts;
        const float4* rp = reinterpret_cast<const float4*>(p.rope + 2 * ((size_t)jt * half + i0));
#pragma unroll
        for (int q = 0; q < 4; ++q) pre[q] = __ldg(rp + q);
      }
    }
    if (FP8)
      for (; conv_done < ntiles && ok; ++conv_done) ok = convert_one(conv_done);
  }

  // ---------------------------------------------------------------- split-K reduction (push model)
  // The 64 * nmt row pairs of this CTA's accumulators are partitioned among the S cluster ranks.
  // Every CTA pushes its partial rows (hi + lo halves already summed) into the owner's receive
  // buffer with plain stores through distributed shared memory, one cluster barrier makes them
  // visible, and each owner adds the S partials of its rows from local shared memory in rank
  // order (deterministic).  No CTA reads another's memory after the barrier, so none waits for
  // its peers before exiting.  The receive buffer overlays the (drained) weight ring and operand
  // tiles, so a first barrier makes sure every peer's MMAs are done before anyone writes.
  const int rmax = 16 * ((n8 + S - 1) / S);            // receive rows per source rank
  const int RST = NT + 4;                               // padded receive row (floats)
  float* recv = reinterpret_cast<float*>(sA);           // [S][rmax][RST]
  float vals[16];
  // the MMA warp arrives only after its accumulators are complete, so passing this barrier means
  // every CTA of the cluster is done with its ring and operand tiles (the receive buffer overlays
  // them); the epilogue warps then observe `done` themselves (already complete: one probe) before
  // reading the accumulators
  tc_fence_before();
  if (S > 1) {
    cluster_arrive_relaxed();
    cluster_wait();
  } else {
    __syncthreads();
  }
  if (warp >= 2) {
    mbar_wait(done, 0, p.status, DEV_ERR_TIMEOUT_MMA);
    tc_fence_after();
    const int quarter = warp & 3;            // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    for (int j = 0; j < nmt; ++j) {
      const int pr = j * 64 + (row >> 1);
      const int oct = pr >> 3;
      const int q = ((oct + 1) * S - 1) / n8;           // owner rank of this row's octet
      const int q0 = 8 * ((q * n8) / S);                 // first pair owned by q
      const int lr = 2 * (pr - q0) + (row & 1);
      float* dst_local = recv + ((size_t)r * rmax + lr) * RST;
      float* dst = S > 1 ? map_peer_w(dst_local, (uint32_t)q) : dst_local;
      // 32 columns (hi and lo) per TMEM round trip
      for (int c0 = 0; c0 < NT; c0 += 32) {
        float vl[16], v2[16], l2[16];
        const bool two = c0 + 16 < NT;          // NT is a multiple of 16: warp-uniform
        const uint32_t ta = tmem_d + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(j * 2 * NT + c0);
        tmem_ld16(ta, vals);
        tmem_ld16(ta + (uint32_t)NT, vl);
        if (two) {
          tmem_ld16(ta + 16u, v2);
          tmem_ld16(ta + (uint32_t)NT + 16u, l2);
        }
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          *reinterpret_cast<float4*>(dst + c0 + c) =
              make_float4(vals[c] + vl[c], vals[c + 1] + vl[c + 1], vals[c + 2] + vl[c + 2], vals[c + 3] + vl[c + 3]);
        if (two) {
#pragma unroll
          for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4*>(dst + c0 + 16 + c) =
                make_float4(v2[c] + l2[c], v2[c + 1] + l2[c + 1], v2[c + 2] + l2[c + 2], v2[c + 3] + l2[c + 3]);
        }
      }
    }
  }
  tc_fence_before();
  if (S > 1) {
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tmem_cols);
  }

  // ---------------------------------------------------------------- epilogue on this CTA's rows
  if (warp >= 2) {
    const int mtid = threadIdx.x - 64;
    const int noct = my_o1 - my_o0;
    float* sq = rstd + NT;                      // [NT][noct] partial sums of squares
    for (int u = mtid; u < my_units; u += kMathThreads) {
      const int col = u % NT, oc = u / NT;
      const int pr0 = (my_o0 + oc) * 8;          // first of the unit's 8 row pairs
      const int j = pr0 >> 6;                    // accumulator (m-tile)
      const int t = nt * NT + col;
      const int o0 = (mt0 + j) * 128 + 2 * (pr0 & 63);   // first of 16 output rows
      const bool valid = (t < p.Ntok) && (o0 < p.O);
      float y[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) y[q] = 0.f;
      for (int s2 = 0; s2 < S; ++s2) {           // rank order: deterministic
        const float* rr = recv + ((size_t)s2 * rmax + 16 * oc) * RST + col;
#pragma unroll
        for (int q = 0; q < 16; ++q) y[q] += rr[(size_t)q * RST];
      }
      const int lr = o0 - mt0 * 128;            // row inside this CTA's staged vectors
      if (ROW_SCALE) {
#pragma unroll
        for (int q = 0; q < 16; ++q) y[q] *= v_wsc[lr + q];
      }
      if (NORM && valid) {
        const float rs = rstd[col];
#pragma unroll
        for (int q = 0; q < 16; ++q) y[q] = fmaf(rs, y[q], v_cshift[lr + q]);
      }
      const int nv = min(16, p.O - o0);          // valid rows of the unit (RESID rows may end early)
      float4 in4[4];
      if (u == mtid && (EPI != EPI_RESID || nv == 16)) {
#pragma unroll
        for (int q = 0; q < 4; ++q) in4[q] = pre[q];
      } else if (valid && EPI == EPI_RESID) {
        float* f = reinterpret_cast<float*>(in4);
#pragma unroll
        for (int q = 0; q < 16; ++q) f[q] = q < nv ? __ldcg(p.h + (size_t)t * p.O + o0 + q) : 0.f;
      } else if (valid && EPI == EPI_QKV && o0 < p.nq * p.hd + p.nkv * p.hd) {
        const int local = o0 < p.nq * p.hd ? o0 : o0 - p.nq * p.hd;
        const float4* rp =
            reinterpret_cast<const float4*>(p.rope + 2 * ((size_t)(t % p.Ts) * (p.hd >> 1) + ((local % p.hd) >> 1)));
#pragma unroll
        for (int q = 0; q < 4; ++q) in4[q] = __ldg(rp + q);
      }
      const float* in = reinterpret_cast<const float*>(in4);
      if (EPI == EPI_RESID) {
        float hsq = 0.f;
        if (valid) {
          float hn[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            hn[q] = q < nv ? fmaf(v_gate[lr + q], y[q], in[q]) : 0.f;
            hsq = fmaf(hn[q], hn[q], hsq);
          }
          if (nv == 16) {
            float4* hp = reinterpret_cast<float4*>(p.h + (size_t)t * p.O + o0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              __stcg(hp + q, make_float4(hn[4 * q], hn[4 * q + 1], hn[4 * q + 2], hn[4 * q + 3]));
          } else {
            for (int q = 0; q < nv; ++q) __stcg(p.h + (size_t)t * p.O + o0 + q, hn[q]);
          }
          if (p.b_next) {
            // 16 consecutive columns = two 16-byte chunks of the next operand (hi and lo tiles)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                __nv_bfloat16 h0, l0, h1, l1;
                const int k = 8 * c + 2 * q;
                split_bf16(hn[k] * (1.f + v_scn[lr + k]), h0, l0);        // zero past the row end
                split_bf16(hn[k + 1] * (1.f + v_scn[lr + k + 1]), h1, l1);
                __nv_bfloat162 hh, ll;
                hh.x = h0;
                hh.y = h1;
                ll.x = l0;
                ll.y = l1;
                hw[q] = *reinterpret_cast<uint32_t*>(&hh);
                lw[q] = *reinterpret_cast<uint32_t*>(&ll);
              }
              const size_t off = operand_offset(t, o0 + 8 * c, NT, p.KBn);
              *reinterpret_cast<uint4*>(p.b_next + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(p.b_next + off + (size_t)NT * 64) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        }
        // one owned octet: this unit is its column's only one, so its sum is the CTA's part and
        // no barrier is needed to collect it
        if (noct == 1) {
          if (t < p.Ntok) p.ss_out[(size_t)(mg * S + r) * p.Ntok + t] = hsq;
        } else {
          sq[col * noct + oc] = hsq;
        }
      } else if (EPI == EPI_SWIGLU) {
        if (valid) {
          // rows (2j, 2j+1) = (gate_j, up_j): 8 consecutive intermediate indices = one 16-byte chunk
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float g0 = y[4 * q], u0 = y[4 * q + 1], g1 = y[4 * q + 2], u1 = y[4 * q + 3];
            __nv_bfloat16 h0, l0, h1, l1;
            split_bf16(g0 / (1.f + __expf(-g0)) * u0, h0, l0);
            split_bf16(g1 / (1.f + __expf(-g1)) * u1, h1, l1);
            __nv_bfloat162 hh, ll;
            hh.x = h0;
            hh.y = h1;
            ll.x = l0;
            ll.y = l1;
            hw[q] = *reinterpret_cast<uint32_t*>(&hh);
            lw[q] = *reinterpret_cast<uint32_t*>(&ll);
          }
          const size_t off = operand_offset(t, o0 >> 1, NT, p.KBm);
          *reinterpret_cast<uint4*>(p.m_out + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(p.m_out + off + (size_t)NT * 64) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      } else {  // EPI_QKV
        if (valid) {
          const int b = t / p.Ts, jt = t % p.Ts;
          const int qd = p.nq * p.hd, kd = p.nkv * p.hd, half = p.hd >> 1;
          if (o0 < qd + kd) {
            // 8 rotary pairs (i0 .. i0+7) of one head: x_i in even rows, x_{i+hd/2} in odd rows
            const bool isq = o0 < qd;
            const int local = isq ? o0 : o0 - qd;
            const int head = local / p.hd, i0 = (local % p.hd) >> 1;
            float r0[8], r1[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float cs = in[2 * q], sn = in[2 * q + 1];
              r0[q] = y[2 * q] * cs - y[2 * q + 1] * sn;
              r1[q] = y[2 * q + 1] * cs + y[2 * q] * sn;
            }
            if (isq) {
              const int rep = p.nq / p.nkv;
              __nv_bfloat16* dst =
                  p.q_out + (((size_t)b * p.nkv + head / rep) * p.Rpad + (head % rep) * p.Ts + jt) * p.hd;
              uint32_t a[4], c[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 x0 = __floats2bfloat162_rn(r0[2 * q], r0[2 * q + 1]);
                __nv_bfloat162 x1 = __floats2bfloat162_rn(r1[2 * q], r1[2 * q + 1]);
                a[q] = *reinterpret_cast<uint32_t*>(&x0);
                c[q] = *reinterpret_cast<uint32_t*>(&x1);
              }
              *reinterpret_cast<uint4*>(dst + i0) = make_uint4(a[0], a[1], a[2], a[3]);
              *reinterpret_cast<uint4*>(dst + i0 + half) = make_uint4(c[0], c[1], c[2], c[3]);
            } else {
              __nv_bfloat16* dst = p.kc + (((size_t)b * p.nkv + head) * p.Lpad + p.P + jt) * p.hd;
              uint32_t a[4], c[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 x0 = __floats2bfloat162_rn(r0[2 * q], r0[2 * q + 1]);
                __nv_bfloat162 x1 = __floats2bfloat162_rn(r1[2 * q], r1[2 * q + 1]);
                a[q] = *reinterpret_cast<uint32_t*>(&x0);
                c[q] = *reinterpret_cast<uint32_t*>(&x1);
              }
              *reinterpret_cast<uint4*>(dst + i0) = make_uint4(a[0], a[1], a[2], a[3]);
              *reinterpret_cast<uint4*>(dst + i0 + half) = make_uint4(c[0], c[1], c[2], c[3]);
            }
          } else {
            const int local = o0 - qd - kd;
            const int head = local / p.hd, d0 = local % p.hd;
            __nv_bfloat16* dst = p.vct + (((size_t)b * p.nkv + head) * p.hd + d0) * p.Lpad + p.P + jt;
#pragma unroll
            for (int q = 0; q < 16; ++q) dst[(size_t)q * p.Lpad] = __float2bfloat16_rn(y[q]);
          }
        }
      }
    }
    if (EPI == EPI_RESID && noct != 1) {
      if (noct > 1) math_bar();
      for (int col = mtid; col < NT; col += kMathThreads) {
        const int t = nt * NT + col;
        if (t < p.Ntok) {
          float acc = 0.f;
          for (int q = 0; q < noct; ++q) acc += sq[col * noct + q];
          p.ss_out[(size_t)(mg * S + r) * p.Ntok + t] = acc;
        }
      }
    }
  }
}

}  // namespace vla
