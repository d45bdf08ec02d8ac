// GQA attention of the action tokens over the cached VLM prefix plus themselves (no mask).
//
// One cluster per (sample b, q head h); its CTAs split the keys (prefix followed by the self
// tokens) into contiguous chunks.  Each CTA computes scores, a warp-shuffle softmax with its
// local max / sum, and a partial P.V; the CTAs then merge their partials through distributed
// shared memory in a fixed order (max-rescaled sums, as in split-K "flash decoding").  The
// prefix part of K / V^T does not depend on the previous kernel and is loaded before
// `griddepcontrol.wait`; the self part (written by the QKV epilogue) and q after it.
// The merged output is written as bf16 straight into the o-projection's operand tiles.
//
// Kept on CUDA cores: at batch 1 the whole attention is ~1-3% of the loop's bytes
// ("AI Infra如何优化VLA" section 算子开发 keeps SDPA on a library kernel for the same reason).
#pragma once
#include "ptx.cuh"

namespace vla {

constexpr int kAttnThreads = 256;

struct AttnParams {
  const __nv_bfloat16* q;    // [Ntok][nq][hd]
  const __nv_bfloat16* kc;   // layer K cache [B][nkv][Lpad][hd]
  const __nv_bfloat16* vct;  // layer V^T cache [B][nkv][hd][Lpad]
  __nv_bfloat16* o_tiles;    // o-proj operand tiles [Nt][KBo][NT][64]
  int nq, nkv, hd, Ts, P, Lpad, Ntok, NT, KBo;
  int S;                     // CTAs per cluster (key chunks)
  int cmax;                  // max keys per chunk
  float scale;               // 1 / sqrt(hd)
  int off_k, off_v, off_s, off_o, off_ml, smem_bytes;
};

template <int HD>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int S = p.S;
  const int g = h / (p.nq / p.nkv);
  const int L = p.P + p.Ts;
  const int j0 = (s * L) / S, j1 = ((s + 1) * L) / S, C = j1 - j0;
  const int Ts = p.Ts;
  constexpr int KST = HD + 2;                 // padded K row (bf16 elements)
  const int VST = p.cmax + 2;                 // padded V^T row (bf16 elements)

  float* qs = reinterpret_cast<float*>(smem);                              // [Ts][HD]
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(smem + p.off_k);   // [cmax][KST]
  __nv_bfloat16* vs = reinterpret_cast<__nv_bfloat16*>(smem + p.off_v);   // [HD][VST]
  float* sc = reinterpret_cast<float*>(smem + p.off_s);                    // [Ts][cmax]
  float* po = reinterpret_cast<float*>(smem + p.off_o);                    // [Ts][HD] partial O
  float* ml = reinterpret_cast<float*>(smem + p.off_ml);                   // [2][Ts] m, l ; [Ts] merge weights ...

  pdl_trigger();
  const __nv_bfloat16* kbase = p.kc + ((size_t)b * p.nkv + g) * p.Lpad * HD;
  const __nv_bfloat16* vbase = p.vct + ((size_t)b * p.nkv + g) * (size_t)HD * p.Lpad;
  auto load_kv = [&](int jb, int je) {
    // K rows jb..je-1 (as 4-byte pairs) and V^T columns jb..je-1
    const int nk = (je - jb) * (HD / 2);
    for (int e = tid; e < nk; e += kAttnThreads) {
      const int jj = jb + e / (HD / 2), d2 = e % (HD / 2);
      *reinterpret_cast<uint32_t*>(&ks[(jj - j0) * KST + 2 * d2]) =
          *reinterpret_cast<const uint32_t*>(&kbase[(size_t)jj * HD + 2 * d2]);
    }
    const int nv = HD * (je - jb);
    for (int e = tid; e < nv; e += kAttnThreads) {
      const int d = e / (je - jb), jj = jb + e % (je - jb);
      vs[d * VST + (jj - j0)] = vbase[(size_t)d * p.Lpad + jj];
    }
  };
  // prefix keys are static during the loop: fetch them before waiting on the QKV kernel
  const int jp = min(j1, p.P);
  if (jp > j0) load_kv(j0, jp);
  pdl_wait();
  if (j1 > max(j0, p.P)) load_kv(max(j0, p.P), j1);
  for (int e = tid; e < Ts * HD; e += kAttnThreads) {
    const int t = e / HD, d = e % HD;
    qs[e] = __bfloat162float(p.q[((size_t)(b * Ts + t) * p.nq + h) * HD + d]);
  }
  __syncthreads();

  // scores: item = (group of 4 tokens, key)
  const int ntg = (Ts + 3) >> 2;
  for (int it = tid; it < ntg * C; it += kAttnThreads) {
    const int jj = it % C, tg = it / C;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16* kr = ks + jj * KST;
#pragma unroll 4
    for (int d = 0; d < HD; d += 2) {
      const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr + d));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = min(tg * 4 + i, Ts - 1);
        const float2 qv = *reinterpret_cast<const float2*>(qs + t * HD + d);
        acc[i] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, acc[i]));
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (tg * 4 + i < Ts) sc[(tg * 4 + i) * p.cmax + jj] = acc[i] * p.scale;
  }
  __syncthreads();

  // warp-shuffle softmax per token row (local to this chunk)
  for (int t = warp; t < Ts; t += kAttnThreads / 32) {
    float mx = -INFINITY;
    for (int jj = lane; jj < C; jj += 32) mx = fmaxf(mx, sc[t * p.cmax + jj]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int jj = lane; jj < C; jj += 32) {
      const float e = __expf(sc[t * p.cmax + jj] - mx);
      sc[t * p.cmax + jj] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      ml[t] = mx;
      ml[Ts + t] = sum;
    }
  }
  __syncthreads();

  // partial O: item = (d, group of 4 tokens)
  for (int it = tid; it < HD * ntg; it += kAttnThreads) {
    const int d = it % HD, tg = it / HD;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16* vr = vs + d * VST;
    for (int jj = 0; jj < C; ++jj) {
      const float v = __bfloat162float(vr[jj]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = min(tg * 4 + i, Ts - 1);
        acc[i] = fmaf(sc[t * p.cmax + jj], v, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (tg * 4 + i < Ts) po[(tg * 4 + i) * HD + d] = acc[i];
  }

  // merge the S partials (fixed order) for this CTA's share of the tokens
  if (S > 1) cluster_sync_all(); else __syncthreads();
  const int t0 = (s * Ts) / S, t1 = ((s + 1) * Ts) / S;
  float* wgt = ml + 2 * Ts;   // [16][Ts] merge weights (S <= 16)
  const uint32_t ml_local = smem_u32(ml), po_local = smem_u32(po);
  // a CTA's own partial is read through the generic window when there is no cluster
  auto ld_peer = [&](uint32_t local_addr, int r) -> float {
    if (S == 1) return *reinterpret_cast<const float*>(smem + (local_addr - smem_u32(smem)));
    return ld_dsmem_f32(mapa_shared(local_addr, (uint32_t)r));
  };
  for (int t = t0 + tid; t < t1; t += kAttnThreads) {
    float mx = -INFINITY;
    for (int r = 0; r < S; ++r) mx = fmaxf(mx, ld_peer(ml_local + t * 4u, r));
    float den = 0.f;
    for (int r = 0; r < S; ++r) {
      const float w = __expf(ld_peer(ml_local + t * 4u, r) - mx);
      wgt[r * Ts + t] = w;
      den += w * ld_peer(ml_local + (Ts + t) * 4u, r);
    }
    for (int r = 0; r < S; ++r) wgt[r * Ts + t] /= den;
  }
  __syncthreads();
  for (int e = tid; e < (t1 - t0) * HD; e += kAttnThreads) {
    const int t = t0 + e / HD, d = e % HD;
    float acc = 0.f;
    for (int r = 0; r < S; ++r)
      acc = fmaf(wgt[r * Ts + t], ld_peer(po_local + (uint32_t)(t * HD + d) * 4u, r), acc);
    const int tok = b * Ts + t;
    const int nt = tok / p.NT, row = tok % p.NT;
    const int k = h * HD + d;
    p.o_tiles[((size_t)nt * p.KBo + (k >> 6)) * p.NT * 64 + sw128_elem_offset(row, k & 63)] = __float2bfloat16_rn(acc);
  }
  if (S > 1) cluster_sync_all(); else __syncthreads();
}

}  // namespace vla
