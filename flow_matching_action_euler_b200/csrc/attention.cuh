// GQA attention of the action tokens over the cached VLM prefix plus themselves (no mask), on
// the tensor cores.
//
// The rep = nq / nkv query heads that share kv head g are stacked into one row set of
// R = rep * Ts rows (row = head_in_group * Ts + token), cut into blocks of 64 rows.  One
// cluster per (sample, kv head, row block); its CTAs split the keys (prefix then self tokens)
// into spans; a CTA walks its span in sub-chunks of CS keys.  Each CTA: 4 warps x 16 rows,
// S = Q K^T with mma.sync m16n8k16 (bf16 in, fp32 accumulate), online exp2 softmax over the
// sub-chunks (row max and sum via quad shuffles, running rescale of the accumulators),
// O += P V with P re-packed from the score registers, then every CTA pushes
// (row max, row sum, partial O) of each row into the shared memory of the row's owner CTA;
// after one cluster barrier owners merge the chunks in rank order (max-rescaled sums, as in
// split-KV "flash decoding") and write the o-projection's hi/lo operand tiles.
// K and V^T of the prefix are static during the loop and are copied before
// `griddepcontrol.wait`; the self rows (written by the QKV epilogue) and q after it.
//
// The pages keep SDPA on a library kernel ("AI Infra如何优化VLA" section 算子开发); here it is a
// hand-written kernel.  At batch 1 attention reads 1-3 % of the loop's bytes but sits on the
// critical path once per layer, so the kernel is built for latency: few, short CTAs.
#pragma once
#include "ptx.cuh"

namespace vla {

constexpr int kAttnThreads = 128;
constexpr int kAttnRows = 64;   // query rows per CTA (4 warps x 16)

struct AttnParams {
  const __nv_bfloat16* q;    // [B][nkv][Rpad][hd] bf16, row = head_in_group * Ts + token (after RoPE)
  const __nv_bfloat16* kc;   // layer K cache [B][nkv][Lpad][hd]
  const __nv_bfloat16* vct;  // layer V^T cache [B][nkv][hd][Lpad]
  __nv_bfloat16* o_tiles;    // o-proj operand tiles [Nt][KBo][2 (hi, lo)][NT][64]
  int nq, nkv, hd, Ts, P, Lpad, Ntok, NT, KBo;
  int S;                     // CTAs per cluster (key chunks), <= 16
  int span;                  // keys per CTA (multiple of 16); CTA c takes [c span, min(L, (c+1) span))
  int nrb;                   // 64-row blocks per kv head
  int Rpad;                  // nrb * 64
  int rpo;                   // rows owned per CTA in the merge = ceil(64 / S)
  float scale;               // 1 / sqrt(hd)
  int off_recv, smem_bytes;   // receive buffer after the block's staging area
};

__device__ __forceinline__ void ldsm_x4(const void* smem_row_addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(smem_row_addr)));
}
__device__ __forceinline__ void mma_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory bytes of one 64-row block: q rows, one sub-chunk of K rows and of V^T columns.
__host__ __device__ constexpr int attn_block_smem(int hd, int cs) {
  return kAttnRows * (hd + 8) * 2 + cs * (hd + 8) * 2 + hd * (cs + 8) * 2;
}

// Partial attention of one 64-row block over the keys [kbeg, kend) of one (sample, kv head):
// 4 warps x 16 rows, `tid` in [0, 128).  `sync()` is a barrier over those 128 threads;
// `before_self()` runs between issuing the prefix copies of the first sub-chunk and the copies
// of anything the loop writes (self K/V rows, q).  Keys past L inside the last 8-column V^T
// copy stay inside the Lpad-long cache rows and meet P = 0; spans are multiples of 16 keys.
// On return `row_dst(r)` (r = 0..63) holds the row's unnormalised O[HD], then (max, sum) in
// base-2 units at [HD], [HD + 1].
template <int HD, int CS, typename Sync, typename BeforeSelf, typename RowDst>
__device__ __forceinline__ void attn_block_partial(uint8_t* smem, const __nv_bfloat16* qbase,
                                                   const __nv_bfloat16* kbase, const __nv_bfloat16* vbase, int P,
                                                   int Lpad, int kbeg, int kend, float scale, int tid, Sync sync,
                                                   BeforeSelf before_self, RowDst row_dst) {
  constexpr int QST = HD + 8, KST = HD + 8, VST = CS + 8;   // padded rows (bf16): conflict-free ldmatrix
  const int warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int nch = kend > kbeg ? (kend - kbeg + CS - 1) / CS : 0;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem);                              // [64][QST]
  __nv_bfloat16* ks = qs + kAttnRows * QST;                                               // [CS][KST]
  __nv_bfloat16* vs = ks + CS * KST;                                                      // [HD][VST]

  // K rows and V^T columns of sub-chunk j0 (part = 0: prefix only, 1: self only, 2: all)
  auto issue_kv = [&](int j0, int part) {
    for (int e = tid; e < CS * (HD / 8); e += kAttnThreads) {
      const int jj = j0 + e / (HD / 8), cc = e % (HD / 8);
      if (jj < kend && (part == 2 || (jj < P) == (part == 0)))
        cp_async16(ks + (jj - j0) * KST + cc * 8, kbase + (size_t)jj * HD + cc * 8);
    }
    for (int e = tid; e < HD * (CS / 8); e += kAttnThreads) {
      const int d = e / (CS / 8), cc = e % (CS / 8);
      const int key0 = j0 + cc * 8;
      if (key0 < kend) {
        if (part == 2 || (key0 + 8 <= P) == (part == 0))
          cp_async16(vs + d * VST + cc * 8, vbase + (size_t)d * Lpad + key0);
      } else if (part != 1) {   // zero columns past the keys: P is 0 there, V must be finite
        *reinterpret_cast<uint4*>(vs + d * VST + cc * 8) = make_uint4(0, 0, 0, 0);
      }
    }
  };
  issue_kv(kbeg, 0);
  cp_async_commit();
  before_self();
  issue_kv(kbeg, 1);
  for (int e = tid; e < kAttnRows * (HD / 8); e += kAttnThreads) {
    const int r = e / (HD / 8), cc = e % (HD / 8);
    cp_async16(qs + r * QST + cc * 8, qbase + (size_t)r * HD + cc * 8);
  }
  cp_async_commit();

  const float sl2 = scale * 1.4426950408889634f;   // 1/sqrt(hd) * log2(e)
  const int arow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows g4 and g4 + 8 of the warp
  float oacc[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;

  for (int ch = 0; ch < nch; ++ch) {
    const int j0 = kbeg + ch * CS, C = min(CS, kend - j0);
    if (ch > 0) {
      sync();   // every warp is done with the previous sub-chunk
      issue_kv(j0, 2);
      cp_async_commit();
    }
    cp_async_wait_all();
    sync();

    // S = Q K^T for the warp's 16 rows
    float sacc[CS / 8][4];
#pragma unroll
    for (int j = 0; j < CS / 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll 4
    for (int kst = 0; kst < HD / 16; ++kst) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(qs + arow * QST + kst * 16 + (lane >> 4) * 8, a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < CS / 16; ++jp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ks + (jp * 16 + (lane & 7) + (lane >> 4) * 8) * KST + kst * 16 + ((lane >> 3) & 1) * 8, b0, b1, b2,
                b3);
        mma_16816(sacc[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_16816(sacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }

    // online softmax in base 2: keys past C are masked (their K rows may hold stale data)
    float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < CS / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 8 + 2 * t4 + (e & 1);
        const float v = key < C ? sacc[j][e] * sl2 : -INFINITY;
        sacc[j][e] = v;
        if (e < 2) x0 = fmaxf(x0, v); else x1 = fmaxf(x1, v);
      }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
    }
    const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);   // finite: C >= 1
    const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);
    m0 = n0;
    m1 = n1;
    l0 *= al0;
    l1 *= al1;
    uint32_t pf[CS / 16][4];
#pragma unroll
    for (int j = 0; j < CS / 8; ++j) {
      const float p0 = exp2f(sacc[j][0] - n0), p1 = exp2f(sacc[j][1] - n0);
      const float p2 = exp2f(sacc[j][2] - n1), p3 = exp2f(sacc[j][3] - n1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      pf[j >> 1][(j & 1) * 2 + 0] = pack_bf16x2(p0, p1);   // row g4:   a0 (keys 16kk..), a2 (keys 16kk+8..)
      pf[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p2, p3);   // row g4+8: a1, a3
    }
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) {
      oacc[n][0] *= al0;
      oacc[n][1] *= al0;
      oacc[n][2] *= al1;
      oacc[n][3] *= al1;
    }

    // O += P V
#pragma unroll
    for (int kk = 0; kk < CS / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(vs + (np * 16 + (lane & 7) + (lane >> 4) * 8) * VST + kk * 16 + ((lane >> 3) & 1) * 8, b0, b1, b2,
                b3);
        mma_16816(oacc[2 * np], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b0, b1);
        mma_16816(oacc[2 * np + 1], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], b2, b3);
      }
    }
  }
  cp_async_wait_all();   // a block left without keys (prefix shorter than planned) still drains its copies
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {   // row sums over the quad (each thread summed its own keys)
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int r0 = warp * 16 + g4, r1 = r0 + 8;
  float* dst0 = row_dst(r0);
  float* dst1 = row_dst(r1);
#pragma unroll
  for (int n = 0; n < HD / 8; ++n) {
    const int d = n * 8 + 2 * t4;
    *reinterpret_cast<float2*>(dst0 + d) = make_float2(oacc[n][0], oacc[n][1]);
    *reinterpret_cast<float2*>(dst1 + d) = make_float2(oacc[n][2], oacc[n][3]);
  }
  if (t4 == 0) {
    *reinterpret_cast<float2*>(dst0 + HD) = make_float2(m0, l0);
    *reinterpret_cast<float2*>(dst1 + HD) = make_float2(m1, l1);
  }
}

// Merge of the S partials (rank order: deterministic) of rows [rbeg, rend) of a 64-row block and
// write of the o-projection's hi/lo operand.  `src(s, r)` points at partial s of block row r
// (O[HD], max, sum); GLOBAL partials written by other SMs are read through L2.
template <int HD, bool GLOBAL, typename Src>
__device__ __forceinline__ void attn_merge_rows(Src src, int S, int rbeg, int rend, int row_base, int R, int Ts,
                                                int b, int kvh, int rep, __nv_bfloat16* o_tiles, int NT, int KBo,
                                                int tid, int nthreads) {
  auto ld1 = [](const float* a) { return GLOBAL ? __ldcg(a) : *a; };
  auto ld4 = [](const float* a) {
    return GLOBAL ? __ldcg(reinterpret_cast<const float4*>(a)) : *reinterpret_cast<const float4*>(a);
  };
  for (int e = tid; e < (rend - rbeg) * (HD / 4); e += nthreads) {
    const int r = rbeg + e / (HD / 4), d = (e % (HD / 4)) * 4;
    const int row = row_base + r;                       // row in this kv head's row set
    if (row >= R) continue;
    float mx = -INFINITY;
    for (int s2 = 0; s2 < S; ++s2) mx = fmaxf(mx, ld1(src(s2, r) + HD));
    float den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s2 = 0; s2 < S; ++s2) {
      const float* sp = src(s2, r);
      const float w = exp2f(ld1(sp + HD) - mx);
      den = fmaf(w, ld1(sp + HD + 1), den);
      const float4 o = ld4(sp + d);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    const float inv = 1.f / den;
    const float v[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
    const int head = kvh * rep + row / Ts, tok = b * Ts + row % Ts;
    const int k = head * HD + d;
    __nv_bfloat16 hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hi[q] = __float2bfloat16_rn(v[q]);
      lo[q] = __float2bfloat16_rn(v[q] - __bfloat162float(hi[q]));
    }
    __nv_bfloat16* base = o_tiles + operand_offset(tok, k, NT, KBo);
    *reinterpret_cast<uint2*>(base) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(base + (size_t)NT * 64) = *reinterpret_cast<const uint2*>(lo);
  }
}

template <int HD, int CS>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int RST = HD + 4;                                 // receive row: O[HD], max, sum
  const int tid = threadIdx.x;
  const int c = blockIdx.x, rb = blockIdx.y % p.nrb, kvh = blockIdx.y / p.nrb, b = blockIdx.z;
  const int S = p.S;
  const int L = p.P + p.Ts;
  const int kbeg = c * p.span, kend = min(L, kbeg + p.span);
  const int rep = p.nq / p.nkv;
  float* recv = reinterpret_cast<float*>(smem + p.off_recv);   // [S][rpo][RST]
  const int rpo = p.rpo;

  pdl_trigger();
  const size_t cache = (size_t)b * p.nkv + kvh;
  attn_block_partial<HD, CS>(
      smem, p.q + (cache * p.Rpad + (size_t)rb * kAttnRows) * HD, p.kc + cache * p.Lpad * HD,
      p.vct + cache * HD * p.Lpad, p.P, p.Lpad, kbeg, kend, p.scale, tid, [] { __syncthreads(); },
      [] { pdl_wait(); },
      [&](int r) {   // push to the row's owner rank
        float* own = recv + ((size_t)c * rpo + (r % rpo)) * RST;
        return S > 1 ? map_peer_w(own, (uint32_t)(r / rpo)) : own;
      });
  if (S > 1) {
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  const int rbeg = c * rpo, rend = min(kAttnRows, rbeg + rpo);
  attn_merge_rows<HD, false>([&](int s2, int r) { return recv + ((size_t)s2 * rpo + (r - rbeg)) * RST; }, S, rbeg,
                             rend, rb * kAttnRows, rep * p.Ts, p.Ts, b, kvh, rep, p.o_tiles, p.NT, p.KBo, tid,
                             kAttnThreads);
}

}  // namespace vla
