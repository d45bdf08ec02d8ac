// GQA attention of the action tokens over the cached VLM prefix plus themselves (no mask).
//
// One cluster per (sample b, q head h); its CTAs split the keys (prefix followed by the self
// tokens) into chunks of `cs` keys (a multiple of 16).  Each CTA stages its K rows, V^T columns
// and q with 16-byte cp.async copies, computes scores, a warp-shuffle softmax with its local
// max / sum, and a partial P.V; the CTAs then merge their partials through distributed shared
// memory in a fixed order (max-rescaled sums, as in split-K "flash decoding").  The prefix part
// of K / V^T does not depend on the previous kernel and is copied before `griddepcontrol.wait`;
// the self part (written by the QKV epilogue) and q after it.  The merged output is written as
// bf16 straight into the o-projection's operand tiles.
//
// Kept on CUDA cores: at batch 1 the whole attention is ~1-3% of the loop's bytes
// ("AI Infra如何优化VLA" section 算子开发 keeps SDPA on a library kernel for the same reason).
// Row strides are padded by 16 bytes so that 16-byte shared loads of consecutive rows hit
// distinct banks.
#pragma once
#include "ptx.cuh"

namespace vla {

constexpr int kAttnThreads = 256;

struct AttnParams {
  const float* q;            // [Ntok][nq][hd] fp32 (after RoPE)
  const __nv_bfloat16* kc;   // layer K cache [B][nkv][Lpad][hd]
  const __nv_bfloat16* vct;  // layer V^T cache [B][nkv][hd][Lpad]
  __nv_bfloat16* o_tiles;    // o-proj operand tiles [Nt][KBo][2 (hi, lo)][NT][64]
  int nq, nkv, hd, Ts, P, Lpad, Ntok, NT, KBo;
  int S;                     // CTAs per cluster (key chunks), <= 16
  int cs;                    // keys per chunk (multiple of 16)
  float scale;               // 1 / sqrt(hd)
  int off_k, off_v, off_s, off_o, off_ml, smem_bytes;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int S = p.S, cs = p.cs, Ts = p.Ts;
  const int g = h / (p.nq / p.nkv);
  const int L = p.P + Ts;
  const int j0 = s * cs, j1 = min(L, j0 + cs), C = max(0, j1 - j0);
  constexpr int QST = HD + 4, KST = HD + 8;   // padded rows (q: fp32, K: bf16 elements)
  const int VST = cs + 8;

  float* qs = reinterpret_cast<float*>(smem);                              // [Ts][QST]
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(smem + p.off_k);   // [cs][KST]
  __nv_bfloat16* vs = reinterpret_cast<__nv_bfloat16*>(smem + p.off_v);   // [HD][VST]
  float* sc = reinterpret_cast<float*>(smem + p.off_s);                    // [Ts][cs]
  float* po = reinterpret_cast<float*>(smem + p.off_o);                    // [Ts][HD] partial O
  float* ml = reinterpret_cast<float*>(smem + p.off_ml);                   // m[Ts], l[Ts], weights[16][Ts]

  pdl_trigger();
  const __nv_bfloat16* kbase = p.kc + ((size_t)b * p.nkv + g) * p.Lpad * HD;
  const __nv_bfloat16* vbase = p.vct + ((size_t)b * p.nkv + g) * (size_t)HD * p.Lpad;
  const int nvc = (C + 7) >> 3;   // 16-byte chunks per V^T row
  auto issue_kv = [&](bool prefix_part) {
    for (int e = tid; e < C * (HD / 8); e += kAttnThreads) {
      const int jj = j0 + e / (HD / 8), c = e % (HD / 8);
      if ((jj < p.P) == prefix_part) cp_async16(ks + (jj - j0) * KST + c * 8, kbase + (size_t)jj * HD + c * 8);
    }
    for (int e = tid; e < HD * nvc; e += kAttnThreads) {
      const int d = e / nvc, c = e % nvc;
      const int key0 = j0 + c * 8;
      if ((key0 + 8 <= p.P) == prefix_part) cp_async16(vs + d * VST + c * 8, vbase + (size_t)d * p.Lpad + key0);
    }
  };
  // prefix keys are static during the loop: fetch them before waiting on the QKV kernel
  issue_kv(true);
  cp_async_commit();
  pdl_wait();
  issue_kv(false);
  for (int e = tid; e < Ts * (HD / 4); e += kAttnThreads) {
    const int t = e / (HD / 4), c = e % (HD / 4);
    cp_async16(qs + t * QST + c * 4, p.q + ((size_t)(b * Ts + t) * p.nq + h) * HD + c * 4);
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();

  // scores: item = (key, group of 4 tokens); 8 dims per 16-byte load
  const int ntg = (Ts + 3) >> 2;
  for (int it = tid; it < ntg * C; it += kAttnThreads) {
    const int jj = it % C, tg = it / C;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint4* kr = reinterpret_cast<const uint4*>(ks + jj * KST);
#pragma unroll 2
    for (int c = 0; c < HD / 8; ++c) {
      float kf[8];
      bf16x8_to_f32(kr[c], kf);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = min(tg * 4 + i, Ts - 1);
        const float4 q0 = *reinterpret_cast<const float4*>(qs + t * QST + c * 8);
        const float4 q1 = *reinterpret_cast<const float4*>(qs + t * QST + c * 8 + 4);
        const float qf[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[i] = fmaf(qf[q], kf[q], acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (tg * 4 + i < Ts) sc[(tg * 4 + i) * cs + jj] = acc[i] * p.scale;
  }
  __syncthreads();

  // warp-shuffle softmax per token row (local to this chunk); entries past C are zeroed
  for (int t = warp; t < Ts; t += kAttnThreads / 32) {
    float mx = -INFINITY;
    for (int jj = lane; jj < C; jj += 32) mx = fmaxf(mx, sc[t * cs + jj]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int jj = lane; jj < cs; jj += 32) {
      const float e = jj < C ? __expf(sc[t * cs + jj] - mx) : 0.f;
      sc[t * cs + jj] = e;
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

  // partial O: item = (d, group of 4 tokens); 8 keys per 16-byte load
  for (int it = tid; it < HD * ntg; it += kAttnThreads) {
    const int d = it % HD, tg = it / HD;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16* vr = vs + d * VST;
    for (int jj = 0; jj < C; jj += 8) {
      float vf[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(vr + jj), vf);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = min(tg * 4 + i, Ts - 1);
        const float4 p0 = *reinterpret_cast<const float4*>(sc + t * cs + jj);
        const float4 p1 = *reinterpret_cast<const float4*>(sc + t * cs + jj + 4);
        acc[i] = fmaf(p0.x, vf[0], acc[i]);
        acc[i] = fmaf(p0.y, vf[1], acc[i]);
        acc[i] = fmaf(p0.z, vf[2], acc[i]);
        acc[i] = fmaf(p0.w, vf[3], acc[i]);
        acc[i] = fmaf(p1.x, vf[4], acc[i]);
        acc[i] = fmaf(p1.y, vf[5], acc[i]);
        acc[i] = fmaf(p1.z, vf[6], acc[i]);
        acc[i] = fmaf(p1.w, vf[7], acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (tg * 4 + i < Ts) po[(tg * 4 + i) * HD + d] = acc[i];
  }

  // merge the S partials (fixed order) for this CTA's share of the tokens
  if (S > 1) cluster_sync_all(); else __syncthreads();
  const int t0 = (s * Ts) / S, t1 = ((s + 1) * Ts) / S;
  float* wgt = ml + 2 * Ts;   // [16][Ts] merge weights
  const uint32_t ml_local = smem_u32(ml), po_local = smem_u32(po);
  for (int t = t0 + tid; t < t1; t += kAttnThreads) {
    float mr[16], lr[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) {
        if (S == 1) {
          mr[r] = ml[t];
          lr[r] = ml[Ts + t];
        } else {
          mr[r] = ld_dsmem_f32(mapa_shared(ml_local + t * 4u, (uint32_t)r));
          lr[r] = ld_dsmem_f32(mapa_shared(ml_local + (Ts + t) * 4u, (uint32_t)r));
        }
      }
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) mx = fmaxf(mx, mr[r]);
    float den = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) {
        mr[r] = __expf(mr[r] - mx);
        den += mr[r] * lr[r];
      }
    const float inv = 1.f / den;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) wgt[r * Ts + t] = mr[r] * inv;
  }
  __syncthreads();
  for (int e = tid; e < (t1 - t0) * (HD / 4); e += kAttnThreads) {
    const int t = t0 + e / (HD / 4), d = (e % (HD / 4)) * 4;
    float4 pr[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) {
        if (S == 1)
          pr[r] = *reinterpret_cast<const float4*>(po + t * HD + d);
        else
          pr[r] = ld_dsmem_f32x4(mapa_shared(po_local + (uint32_t)(t * HD + d) * 4u, (uint32_t)r));
      }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < S) {
        const float w = wgt[r * Ts + t];
        acc.x = fmaf(w, pr[r].x, acc.x);
        acc.y = fmaf(w, pr[r].y, acc.y);
        acc.z = fmaf(w, pr[r].z, acc.z);
        acc.w = fmaf(w, pr[r].w, acc.w);
      }
    const int tok = b * Ts + t;
    const int nt = tok / p.NT, row = tok % p.NT;
    const int k = h * HD + d;
    // hi / lo bf16 pair per value, 4 consecutive columns inside one 16-byte chunk
    const float v[4] = {acc.x, acc.y, acc.z, acc.w};
    __nv_bfloat16 hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hi[q] = __float2bfloat16_rn(v[q]);
      lo[q] = __float2bfloat16_rn(v[q] - __bfloat162float(hi[q]));
    }
    __nv_bfloat16* base = p.o_tiles + ((size_t)nt * p.KBo + (k >> 6)) * 2 * p.NT * 64 + sw128_elem_offset(row, k & 63);
    *reinterpret_cast<uint2*>(base) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(base + (size_t)p.NT * 64) = *reinterpret_cast<const uint2*>(lo);
  }
  // peers read this CTA's partials: exit only after every CTA has finished reading (the relaxed
  // arrive does not wait for this CTA's global stores)
  if (S > 1) {
    cluster_arrive_relaxed();
    cluster_wait();
  }
}

}  // namespace vla
