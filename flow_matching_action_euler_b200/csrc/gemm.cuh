// Skinny weight-streaming GEMM for the action expert's linears, y[t][o] = sum_k W[o][k] x[t][k].
//
// Swap-AB: the weight's output rows are the tcgen05 M side (128 rows per tile) and the few
// tokens (batch x self tokens, padded to a multiple of 16) are the N side, so one M=128 x
// N=NT x K=16 MMA consumes a whole 128-row strip of weights.  At batch 1 the loop is bound by
// the weight stream from HBM ("跨XPU平台表征视觉-语言-动作模型" section 4.2: the action expert is
// memory-bound), so the kernel is organised around keeping that stream full:
//
//  * weights are pre-packed at create time into 16 KB tiles (128 rows x 64 bf16, or 128 rows x
//    128 e4m3) already laid out in the 128-byte swizzle the MMA reads, stored [m-tile][k-block]
//    so every CTA's share is one contiguous range, fetched with 1-D bulk copies (TMA engine);
//  * the producer warp issues those copies before `griddepcontrol.wait`, i.e. while the previous
//    kernel of the loop is still running (programmatic dependent launch);
//  * split-K across the CTAs of a thread-block cluster, reduced through distributed shared
//    memory in a fixed order (deterministic, no float atomics);
//  * fused B-operand prologue (RMSNorm + adaLN modulate of the fp32 residual, "AI Infra如何优化VLA"
//    section 算子开发) and fused epilogues: RoPE (half-split rotation) writing q and the layer's
//    K / V^T caches, SwiGLU (section 算子融合) writing the down GEMM's operand, and the gated
//    residual add writing h plus per-row partial sums of squares for the next RMSNorm.
//
// Warp roles (320 threads): warp 0 = bulk-copy producer, warp 1 = MMA issuer (and TMEM owner),
// warps 2..9 = math warps (B prologue, fp8 -> bf16 conversion, TMEM read-out, epilogue).
#pragma once
#include "ptx.cuh"

namespace vla {

enum EpiKind : int { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };
enum BMode : int { B_NORM = 0, B_TILES = 1 };

constexpr int kGemmThreads = 320;
constexpr int kMathThreads = 256;
constexpr int kTileBytes = 16384;      // one packed weight tile
constexpr int kConvStages = 2;         // fp8 path: converted bf16 A stages (2 x 16 KB each)

struct GemmParams {
  // ---- A operand (packed weights)
  const uint8_t* w;        // tiles [Mt][KBt][16 KB]
  const float* wscale;     // fp8: scale per packed row (else nullptr)
  int Mt;                  // 128-row output tiles
  int KBt;                 // weight tiles along K (64 wide for bf16, 128 wide for fp8)
  int K;                   // logical reduction length
  int S;                   // K splits = cluster size along x
  int stages;              // weight-tile ring depth
  // ---- tokens
  int Ntok;                // valid token rows
  int NT;                  // token rows per n-tile (multiple of 16, <= 256)
  int KB;                  // 64-wide k-blocks of the B operand = ceil(K / 64)
  // ---- B operand
  const __nv_bfloat16* act;  // B_TILES: [Nt][KB][NT][64] swizzled operand tiles
  const float* h;            // B_NORM: residual [Ntok][K]
  const float* ss;           // B_NORM: partial sums of squares [ss_parts][Ntok]
  int ss_parts;
  const float* shift;        // B_NORM: [K]
  const float* scale;        // B_NORM: [K]
  float eps;
  // ---- epilogue
  int O;                     // packed output rows
  float* h_out;              // RESID: residual [Ntok][O] updated in place
  const float* gate;         // RESID: [O]
  float* ss_out;             // RESID: [Mt * S][Ntok]
  __nv_bfloat16* m_out;      // SWIGLU: down-GEMM operand tiles [Nt][KBm][NT][64]
  int KBm;
  __nv_bfloat16* q_out;      // QKV: q [Ntok][nq][hd]
  __nv_bfloat16* kc;         // QKV: layer K cache [B][nkv][Lpad][hd]
  __nv_bfloat16* vct;        // QKV: layer V^T cache [B][nkv][hd][Lpad]
  const float* rope;         // QKV: [Ts][hd/2][2] (cos, sin) for positions P + j
  int nq, nkv, hd, Ts, P, Lpad;
  unsigned* status;
  // ---- shared-memory layout (bytes from the 1024-aligned base)
  int off_b, off_conv, off_bar, off_misc, kmax, smem_bytes;
};

__device__ __forceinline__ void math_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <int EPI, int BMODE, bool FP8>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_stream_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S;
  const int r = blockIdx.x;          // rank inside the cluster (cluster dims = (S,1,1), grid.x = S)
  const int mt = blockIdx.y, nt = blockIdx.z;
  const int kt0 = (r * p.KBt) / S, kt1 = ((r + 1) * p.KBt) / S, nkt = kt1 - kt0;
  constexpr int KPT = FP8 ? 2 : 1;   // 64-wide k-blocks per weight tile
  const int kb0 = kt0 * KPT;
  const int kb1 = min(kt1 * KPT, p.KB);
  const int NT = p.NT;

  uint8_t* sA = smem;                                     // weight ring (and later the reduction buffer)
  uint8_t* sB = smem + p.off_b;                           // B operand tiles for this CTA's k-range
  uint8_t* sC = smem + p.off_conv;                        // fp8: converted bf16 A stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* full = bars;                                  // [stages]
  uint64_t* empty = bars + p.stages;                      // [stages]
  uint64_t* bfull = bars + 2 * p.stages;
  uint64_t* done = bfull + 1;
  uint64_t* cfull = done + 1;                             // [kConvStages]
  uint64_t* cempty = cfull + kConvStages;                 // [kConvStages]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + kConvStages);
  float* s_shift = reinterpret_cast<float*>(smem + p.off_misc);   // [kmax] modulation slice of this CTA
  float* s_scale = s_shift + p.kmax;                              // [kmax]
  float* rpart = s_scale + p.kmax;                                // [256] partial sums of squares
  float* rstd = rpart + kMathThreads;                             // [NT]

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], FP8 ? kMathThreads : 1);
    }
    mbar_init(bfull, BMODE == B_NORM ? kMathThreads : 1);
    mbar_init(done, 1);
    for (int i = 0; i < kConvStages; ++i) {
      mbar_init(&cfull[i], kMathThreads);
      mbar_init(&cempty[i], 1);
    }
    fence_mbar_init();
  }
  const int tmem_cols = NT <= 32 ? 32 : (NT <= 64 ? 64 : (NT <= 128 ? 128 : 256));
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer: weight stream
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint8_t* src = p.w + ((size_t)mt * p.KBt + kt0) * kTileBytes;
      const int prefill = min(nkt, p.stages);
      // the first ring's worth of weights does not depend on the previous kernel
      for (int i = 0; i < prefill; ++i) {
        mbar_arrive_expect_tx(&full[i], kTileBytes);
        bulk_g2s(sA + (size_t)i * kTileBytes, src + (size_t)i * kTileBytes, kTileBytes, &full[i], pol);
      }
      if (BMODE == B_TILES) {
        // activation tiles are produced by the previous kernel: only after its completion
        pdl_wait();
        const uint32_t bytes = (uint32_t)(kb1 - kb0) * NT * 128u;
        mbar_arrive_expect_tx(bfull, bytes);
        bulk_g2s(sB, p.act + ((size_t)nt * p.KB + kb0) * NT * 64, bytes, bfull, policy_evict_last());
      }
      for (int i = prefill; i < nkt; ++i) {
        const int s = i % p.stages;
        if (!mbar_wait(&empty[s], ((i / p.stages) - 1) & 1, p.status, DEV_ERR_TIMEOUT_TMA)) break;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        bulk_g2s(sA + (size_t)s * kTileBytes, src + (size_t)i * kTileBytes, kTileBytes, &full[s], pol);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, NT);
      bool ok = mbar_wait(bfull, 0, p.status, DEV_ERR_TIMEOUT_TMA);
      const uint32_t aBase = smem_u32(FP8 ? sC : sA), bBase = smem_u32(sB);
      uint32_t acc = 0;
      for (int i = 0; i < nkt && ok; ++i) {
        if (!FP8) {
          const int s = i % p.stages;
          ok = mbar_wait(&full[s], (i / p.stages) & 1, p.status, DEV_ERR_TIMEOUT_TMA);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(tmem_d, sw128_desc(aBase + s * kTileBytes + kk * 32),
                     sw128_desc(bBase + (uint32_t)i * NT * 128u + kk * 32), idesc, acc);
            acc = 1;
          }
          mma_commit(&empty[s]);
        } else {
          const int c = i % kConvStages;
          ok = mbar_wait(&cfull[c], (i / kConvStages) & 1, p.status, DEV_ERR_TIMEOUT_CONV);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int lkb = i * 2 + half;                       // local 64-wide k-block
            if (kb0 + lkb >= kb1) break;                        // ragged K tail
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_bf16(tmem_d, sw128_desc(aBase + (c * 2 + half) * kTileBytes + kk * 32),
                       sw128_desc(bBase + (uint32_t)lkb * NT * 128u + kk * 32), idesc, acc);
              acc = 1;
            }
          }
          mma_commit(&cempty[c]);
        }
      }
      mma_commit(done);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    const int mtid = threadIdx.x - 64;   // 0..255
    int conv_done = 0;
    auto convert_one = [&](int i) -> bool {
      // fp8 tile (128 rows x 128 B, swizzled by 16 B chunks) -> two bf16 SW128 tiles
      const int s = i % p.stages, c = i % kConvStages;
      if (!mbar_wait(&full[s], (i / p.stages) & 1, p.status, DEV_ERR_TIMEOUT_TMA)) return false;
      if (i >= kConvStages && !mbar_wait(&cempty[c], ((i / kConvStages) - 1) & 1, p.status, DEV_ERR_TIMEOUT_CONV))
        return false;
      const uint8_t* src = sA + (size_t)s * kTileBytes;
      uint8_t* dst = sC + (size_t)c * 2 * kTileBytes;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int idx = mtid + j * kMathThreads;   // 0..1023: (row, fp8 chunk)
        const int row = idx >> 3, ch = idx & 7;
        const uint4 raw = *reinterpret_cast<const uint4*>(src + sw128_chunk_byte(row, ch));
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          o[2 * q] = e4m3x2_to_bf16x2((uint16_t)(w4[q] & 0xFFFFu));
          o[2 * q + 1] = e4m3x2_to_bf16x2((uint16_t)(w4[q] >> 16));
        }
        const int half = ch >> 2;                // which 64-wide bf16 tile
        const int bch = (ch & 3) * 2;            // first bf16 chunk (8 elements) inside it
        uint8_t* t = dst + half * kTileBytes;
        *reinterpret_cast<uint4*>(t + sw128_chunk_byte(row, bch)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(t + sw128_chunk_byte(row, bch + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&cfull[c]);
      mbar_arrive(&empty[s]);
      return true;
    };
    bool ok = true;
    if (FP8) {
      // weights do not depend on the previous kernel: convert the first stages before waiting
      const int pre = min(nkt, kConvStages);
      for (; conv_done < pre && ok; ++conv_done) ok = convert_one(conv_done);
    }
    const int nkb = kb1 - kb0;
    if (BMODE == B_NORM) {
      // the modulation vectors are input-independent: stage this CTA's slice before waiting
      for (int i = mtid; i < nkb * 64; i += kMathThreads) {
        const int k = kb0 * 64 + i;
        s_shift[i] = k < p.K ? __ldg(p.shift + k) : 0.f;
        s_scale[i] = k < p.K ? __ldg(p.scale + k) : 0.f;
      }
    }
    pdl_wait();
    if (BMODE == B_NORM) {
      // rstd per token row from the producers' partial sums of squares: G threads per row each
      // take every G-th part, then the G partials are added in a fixed order (deterministic)
      const int G = NT >= kMathThreads ? 1 : kMathThreads / NT;
      {
        const int row = mtid / G, g = mtid % G;
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
      }
      math_bar();
      for (int row = mtid; row < NT; row += kMathThreads) {
        float acc = 0.f;
        if (NT >= kMathThreads) {
          acc = rpart[row];   // G == 1: one thread per row already summed everything
        } else {
          for (int g = 0; g < G; ++g) acc += rpart[row * G + g];
        }
        rstd[row] = rsqrtf(acc / (float)p.K + p.eps);
      }
      math_bar();
      // u = rms(h) * (1 + scale) + shift -> bf16, written straight into the swizzled B tiles;
      // loads are issued in batches of 4 chunks so their latencies overlap
      const int nchunks = NT * nkb * 8;
      for (int e0 = mtid; e0 < nchunks; e0 += 4 * kMathThreads) {
        float4 hv[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * kMathThreads;
          const int ch = e & 7, rest = e >> 3;
          const int row = rest % NT, lk = rest / NT;
          const int t = nt * NT + row;
          const int k = (kb0 + lk) * 64 + ch * 8;
          if (e < nchunks && t < p.Ntok && k < p.K) {
            const float4* hp = reinterpret_cast<const float4*>(p.h + (size_t)t * p.K + k);
            hv[u][0] = __ldcg(hp);
            hv[u][1] = __ldcg(hp + 1);
          } else {
            hv[u][0] = make_float4(0.f, 0.f, 0.f, 0.f);
            hv[u][1] = hv[u][0];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * kMathThreads;
          if (e >= nchunks) break;
          const int ch = e & 7, rest = e >> 3;
          const int row = rest % NT, lk = rest / NT;
          const int t = nt * NT + row;
          const int kl = lk * 64 + ch * 8;
          const int k = kb0 * 64 + kl;
          uint4 packed = make_uint4(0, 0, 0, 0);
          if (t < p.Ntok && k < p.K) {
            const float rs = rstd[row];
            const float hvals[8] = {hv[u][0].x, hv[u][0].y, hv[u][0].z, hv[u][0].w,
                                    hv[u][1].x, hv[u][1].y, hv[u][1].z, hv[u][1].w};
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float v0 = hvals[2 * q] * rs * (1.f + s_scale[kl + 2 * q]) + s_shift[kl + 2 * q];
              const float v1 = hvals[2 * q + 1] * rs * (1.f + s_scale[kl + 2 * q + 1]) + s_shift[kl + 2 * q + 1];
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
              w4[q] = *reinterpret_cast<uint32_t*>(&b2);
            }
            packed = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          *reinterpret_cast<uint4*>(sB + (size_t)lk * NT * 128 + sw128_chunk_byte(row, ch)) = packed;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bfull);
    }
    if (FP8)
      for (; conv_done < nkt && ok; ++conv_done) ok = convert_one(conv_done);
  }

  // ---------------------------------------------------------------- accumulator -> shared memory
  float* red = reinterpret_cast<float*>(sA);   // [NT][128] fp32 (weight ring is drained by now)
  if (warp >= 2) {
    const bool ok = mbar_wait(done, 0, p.status, DEV_ERR_TIMEOUT_MMA);
    tc_fence_after();
    const int quarter = warp & 3;            // TMEM lanes this warp may access
    const int colhalf = (warp - 2) >> 2;     // two warps per lane quarter split the columns
    const int row = quarter * 32 + lane;
    const int ncol = NT / 2;
    for (int c0 = colhalf * ncol; c0 < (colhalf + 1) * ncol; c0 += 16) {
      float v[16];
      tmem_ld16(tmem_d + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) red[(c0 + j) * 128 + row] = ok ? v[j] : 0.f;
    }
  }
  tc_fence_before();
  if (S > 1) cluster_sync_all(); else __syncthreads();

  // ---------------------------------------------------------------- split-K reduction + epilogue
  if (warp >= 2) {
    const int mtid = threadIdx.x - 64;
    const int p0 = (r * 64) / S, p1 = ((r + 1) * 64) / S, npairs = p1 - p0;
    const uint32_t red_local = smem_u32(red);
    float* sq = reinterpret_cast<float*>(sB);   // [NT][npairs] (B tiles are consumed by now)
    for (int e = mtid; e < npairs * NT; e += kMathThreads) {
      const int col = e / npairs, pr = p0 + e % npairs;
      const int t = nt * NT + col;
      const int o0 = mt * 128 + 2 * pr;
      float y0 = 0.f, y1 = 0.f;
      const uint32_t off = (uint32_t)(col * 128 + 2 * pr) * 4u;
      if (S > 1) {
        // all S remote loads in flight first, then the sum in rank order (deterministic)
        float2 part[16];
#pragma unroll
        for (int s = 0; s < 16; ++s)
          if (s < S) part[s] = ld_dsmem_f32x2(mapa_shared(red_local + off, (uint32_t)s));
#pragma unroll
        for (int s = 0; s < 16; ++s)
          if (s < S) {
            y0 += part[s].x;
            y1 += part[s].y;
          }
      } else {
        y0 = red[col * 128 + 2 * pr];
        y1 = red[col * 128 + 2 * pr + 1];
      }
      if (FP8) {
        if (o0 < p.O) y0 *= p.wscale[o0];
        if (o0 + 1 < p.O) y1 *= p.wscale[o0 + 1];
      }
      const bool valid = (t < p.Ntok) && (o0 < p.O);
      if (EPI == EPI_RESID) {
        float hsq = 0.f;
        if (valid) {
          float2* hp = reinterpret_cast<float2*>(p.h_out + (size_t)t * p.O + o0);
          const float2 ho = __ldcg(hp);
          const float hn0 = ho.x + __ldg(p.gate + o0) * y0;
          const float hn1 = ho.y + __ldg(p.gate + o0 + 1) * y1;
          __stcg(hp, make_float2(hn0, hn1));
          hsq = hn0 * hn0 + hn1 * hn1;
        }
        sq[col * npairs + (e % npairs)] = hsq;
      } else if (EPI == EPI_SWIGLU) {
        if (valid) {
          const int j = o0 >> 1;                 // intermediate index: rows (2j, 2j+1) = (gate_j, up_j)
          const float g = y0;
          const float m = g / (1.f + __expf(-g)) * y1;
          const int kb = j >> 6, c = j & 63;
          p.m_out[((size_t)nt * p.KBm + kb) * NT * 64 + sw128_elem_offset(col, c)] = __float2bfloat16_rn(m);
        }
      } else {  // EPI_QKV
        if (valid) {
          const int b = t / p.Ts, jt = t % p.Ts;
          const int qd = p.nq * p.hd, kd = p.nkv * p.hd, half = p.hd >> 1;
          if (o0 < qd + kd) {
            const bool isq = o0 < qd;
            const int local = isq ? o0 : o0 - qd;
            const int head = local / p.hd, i = (local % p.hd) >> 1;  // pair i rotates (x_i, x_{i+hd/2})
            const float2 cs = reinterpret_cast<const float2*>(p.rope)[(size_t)jt * half + i];
            const float r0 = y0 * cs.x - y1 * cs.y;
            const float r1 = y1 * cs.x + y0 * cs.y;
            __nv_bfloat16* dst;
            if (isq) {
              dst = p.q_out + ((size_t)t * p.nq + head) * p.hd;
            } else {
              dst = p.kc + (((size_t)b * p.nkv + head) * p.Lpad + p.P + jt) * p.hd;
            }
            dst[i] = __float2bfloat16_rn(r0);
            dst[i + half] = __float2bfloat16_rn(r1);
          } else {
            const int local = o0 - qd - kd;
            const int head = local / p.hd, d = local % p.hd;
            __nv_bfloat16* dst = p.vct + (((size_t)b * p.nkv + head) * p.hd + d) * p.Lpad + p.P + jt;
            dst[0] = __float2bfloat16_rn(y0);
            dst[p.Lpad] = __float2bfloat16_rn(y1);
          }
        }
      }
    }
    if (EPI == EPI_RESID) {
      math_bar();
      for (int col = mtid; col < NT; col += kMathThreads) {
        const int t = nt * NT + col;
        if (t < p.Ntok) {
          float acc = 0.f;
          for (int q = 0; q < npairs; ++q) acc += sq[col * npairs + q];
          p.ss_out[(size_t)(mt * S + r) * p.Ntok + t] = acc;
        }
      }
    }
  }
  if (S > 1) cluster_sync_all(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, tmem_cols);
  }
}

}  // namespace vla
