// Small kernels around the GEMMs: the per-step tail (final RMSNorm + adaLN modulate, action
// out-projection, Euler update, next step's in-projection), the input-independent tables
// (adaLN modulation per (step, layer), RoPE cos/sin for the self-token positions), weight
// packing / fp8 quantisation at create time, and the prefix-cache layout at set_prefix time.
#pragma once
#include "ptx.cuh"

namespace vla {

constexpr int kTailThreads = 256;
constexpr int kTileBytesPack = 16384;   // one packed weight tile (same as the GEMM's)
constexpr int kMaxAction = 64;

// ---------------------------------------------------------------- step tail / in-projection
// One CTA per token row t = b * Ts + j.  Row j < has_state is the state token (not denoised),
// the others are action tokens a = j - has_state.
//  do_out: v = W_out (rms(h) * (1 + sc_f) + sh_f) + b_out ;  x += dt * v   (flow-matching Euler,
//          "AI Infra如何优化VLA" section 整体方案)
//  do_in : h = W_in x + b_in (state row: the cached W_st s + b_st), plus the row's sum of squares
struct TailParams {
  float* h;                 // [Ntok][H]
  const float* ss;          // [ss_parts][Ntok]
  int ss_parts;
  float* ss_out;            // [1][Ntok]
  const float* shift_f;     // [H]
  const float* scale_f;     // [H]
  const __nv_bfloat16* w_out;  // [A][H]
  const __nv_bfloat16* b_out;  // [A]
  const __nv_bfloat16* w_in;   // [H][A]
  const __nv_bfloat16* b_in;   // [H]
  const float* h_state0;    // [B][H]
  const __nv_bfloat16* noise;  // [B][T][A] (init only)
  float* x;                 // [B][T][A]
  float* out;               // [B][T][A] copy of x after the update (or nullptr)
  float* v_out;             // [B][T][A] velocity (debug, or nullptr)
  __nv_bfloat16* b_out_tiles;  // next QKV GEMM's operand tiles [Nt][KBh][2][NT][64]
  const float* sc_next;     // [H] modulation scale of that GEMM (layer 0 of the next step)
  int NT, KBh;
  float dt, eps;
  int H, A, T, Ts, has_state, Ntok;
  int do_out, do_in, init_from_noise;
};

__device__ __forceinline__ void store_operand(__nv_bfloat16* tiles, int t, int k, int NT, int KB, float x) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
  const size_t off = operand_offset(t, k, NT, KB);
  tiles[off] = hi;
  tiles[off + (size_t)NT * 64] = lo;
}

__global__ void __launch_bounds__(kTailThreads) tail_kernel(const __grid_constant__ TailParams p) {
  __shared__ float vsh[kMaxAction];
  __shared__ float xs[kMaxAction];
  __shared__ float red[kTailThreads / 32];
  __shared__ float rs_sh;
  const int t = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = t / p.Ts, j = t % p.Ts;
  const bool is_state = j < p.has_state;
  const int a_row = j - p.has_state;
  const int H = p.H, A = p.A;
  pdl_trigger();
  pdl_wait();
  float* hrow = p.h + (size_t)t * H;
  float* xrow = is_state ? nullptr : p.x + ((size_t)b * p.T + a_row) * A;
  if (!is_state && p.init_from_noise && tid < A)
    xrow[tid] = __bfloat162float(p.noise[((size_t)b * p.T + a_row) * A + tid]);
  if (!is_state && p.do_out) {
    if (warp == 0) {   // rstd from the down GEMM's partial sums of squares (fixed order)
      float acc = 0.f;
      for (int q = lane; q < p.ss_parts; q += 32) acc += __ldcg(p.ss + (size_t)q * p.Ntok + t);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) rs_sh = rsqrtf(acc / (float)H + p.eps);
    }
    __syncthreads();
    const float rs = rs_sh;
    // v[a] = W_out[a] . (rms(h) (1 + sc_f) + sh_f) + b_out[a]: one warp per output, lanes over k
    for (int a = warp; a < A; a += kTailThreads / 32) {
      float acc = 0.f;
      for (int k = lane; k < H; k += 32) {
        const float u = __ldcg(hrow + k) * rs * (1.f + __ldg(p.scale_f + k)) + __ldg(p.shift_f + k);
        acc = fmaf(__bfloat162float(p.w_out[(size_t)a * H + k]), u, acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) vsh[a] = acc + __bfloat162float(p.b_out[a]);
    }
    __syncthreads();
    if (tid < A) {
      const float v = vsh[tid];
      if (p.v_out) p.v_out[((size_t)b * p.T + a_row) * A + tid] = v;
      const float xn = xrow[tid] + p.dt * v;
      xrow[tid] = xn;
      if (p.out) p.out[((size_t)b * p.T + a_row) * A + tid] = xn;
    }
  }
  if (!p.do_in) return;
  __syncthreads();
  if (!is_state && tid < A) xs[tid] = xrow[tid];
  __syncthreads();
  // next step's self-token row: W_in x + b_in (action rows) or the cached state projection
  float sq = 0.f;
  for (int o = tid; o < H; o += kTailThreads) {
    float v;
    if (is_state) {
      v = p.h_state0[(size_t)b * H + o];
    } else {
      v = __bfloat162float(p.b_in[o]);
      for (int a = 0; a < A; ++a) v = fmaf(__bfloat162float(p.w_in[(size_t)o * A + a]), xs[a], v);
    }
    hrow[o] = v;
    sq = fmaf(v, v, sq);
    store_operand(p.b_out_tiles, t, o, p.NT, p.KBh, v * (1.f + __ldg(p.sc_next + o)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0) red[warp] = sq;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < kTailThreads / 32; ++w) s += red[w];
    p.ss_out[t] = s;
  }
}

// ---------------------------------------------------------------- input-independent tables
// c_k = SiLU(temb(t_k)), temb(t) = [cos(a_i), sin(a_i)], a_i = 1000 t 10000^(-i/half), in double.
__global__ void temb_kernel(const double* __restrict__ ts, double* c, int dt_dim) {
  const int k = blockIdx.x, half = dt_dim / 2;
  const double t = ts[k];
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double a = 1000.0 * t * exp(-log(10000.0) * (double)i / (double)half);
    const double cs = cos(a), sn = sin(a);
    c[(size_t)k * dt_dim + i] = cs / (1.0 + exp(-cs));
    c[(size_t)k * dt_dim + half + i] = sn / (1.0 + exp(-sn));
  }
}

// table[k][row] = W[row] . c_k + b[row] for rows of one adaLN weight (one warp per row).
__global__ void adaln_table_kernel(const __nv_bfloat16* __restrict__ w, const __nv_bfloat16* __restrict__ bias,
                                   const double* __restrict__ c, int rows, int dt_dim, int steps, float* out,
                                   size_t step_stride) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  for (int k = 0; k < steps; ++k) {
    double acc = 0.0;
    for (int i = lane; i < dt_dim; i += 32) acc += (double)__bfloat162float(w[(size_t)row * dt_dim + i]) * c[(size_t)k * dt_dim + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[(size_t)k * step_stride + row] = (float)(acc + (double)__bfloat162float(bias[row]));
  }
}

// rope[j][i] = (cos, sin)(theta), theta = (P + j) * base^(-2i/hd), in double.
__global__ void rope_table_kernel(float2* rope, int Ts, int P, int hd, double base) {
  const int half = hd / 2;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < Ts * half; e += gridDim.x * blockDim.x) {
    const int j = e / half, i = e % half;
    const double th = (double)(P + j) * pow(base, -2.0 * (double)i / (double)hd);
    rope[e] = make_float2((float)cos(th), (float)sin(th));
  }
}

// h_state0[b] = W_st s_b + b_st
__global__ void state_proj_kernel(const __nv_bfloat16* w, const __nv_bfloat16* bias, const __nv_bfloat16* state,
                                  float* out, int H, int A) {
  const int b = blockIdx.y;
  for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < H; o += gridDim.x * blockDim.x) {
    float v = __bfloat162float(bias[o]);
    for (int a = 0; a < A; ++a)
      v = fmaf(__bfloat162float(w[(size_t)o * A + a]), __bfloat162float(state[(size_t)b * A + a]), v);
    out[(size_t)b * H + o] = v;
  }
}

// ---------------------------------------------------------------- weight packing (create time)
// Gather source rows (row pointers, nullptr = zero row) into 16 KB bf16 tiles [Mt][KB][128][64]
// in the 128-byte swizzle layout.  One thread per 16-byte chunk.
__global__ void pack_bf16_kernel(const __nv_bfloat16* const* __restrict__ rows, int K, int Mt, int KB,
                                 uint8_t* __restrict__ dst) {
  const size_t total = (size_t)Mt * KB * 128 * 8;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int ch = (int)(e & 7);
    const int r = (int)((e >> 3) & 127);
    const size_t tile = e >> 10;
    const int kb = (int)(tile % KB), mt = (int)(tile / KB);
    const __nv_bfloat16* src = rows[mt * 128 + r];
    const int k0 = kb * 64 + ch * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (src && k0 < K) v = *reinterpret_cast<const uint4*>(src + k0);
    *reinterpret_cast<uint4*>(dst + tile * kTileBytesPack + sw128_chunk_byte(r, ch)) = v;
  }
}

// Per-output-channel e4m3 quantisation (one warp per packed row):
// scale = max|w| / 448 (IEEE division; 1 for a zero row), code = e4m3_rn_sat(w / scale).
// Codes go to 16 KB tiles [Mt][KB8][128][128 B], 16-byte chunks swizzled like the bf16 tiles.
__global__ void quant_e4m3_kernel(const __nv_bfloat16* const* __restrict__ rows, int K, int Mt, int KB8,
                                  uint8_t* __restrict__ dst, float* __restrict__ scales) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= Mt * 128) return;
  const __nv_bfloat16* src = rows[row];
  float amax = 0.f;
  if (src)
    for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(__bfloat162float(src[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sc = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
  if (lane == 0) scales[row] = sc;
  const int mt = row >> 7, r = row & 127;
  for (int c = lane; c < KB8 * 8; c += 32) {            // 16-element chunks along K
    const int kb = c >> 3, ch = c & 7, k0 = c * 16;
    uint32_t word[4] = {0, 0, 0, 0};
    if (src) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int k = k0 + 2 * q;
        const float lo = (k < K) ? __fdiv_rn(__bfloat162float(src[k]), sc) : 0.f;
        const float hi = (k + 1 < K) ? __fdiv_rn(__bfloat162float(src[k + 1]), sc) : 0.f;
        word[q >> 1] |= (uint32_t)f32x2_to_e4m3x2(lo, hi) << ((q & 1) * 16);
      }
    }
    *reinterpret_cast<uint4*>(dst + ((size_t)mt * KB8 + kb) * kTileBytesPack + sw128_chunk_byte(r, ch)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// Row-wise symmetric int8 packing: scale = max|w| / 127 (1 for a zero row), code =
// round-to-nearest-even(w / scale) clamped to [-127, 127] (code -128 unused), laid out like the
// e4m3 tiles (128 rows x 128 codes per 16 KB tile, 16-byte chunks swizzled).
__global__ void quant_int8_kernel(const __nv_bfloat16* const* __restrict__ rows, int K, int Mt, int KB8,
                                  uint8_t* __restrict__ dst, float* __restrict__ scales) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= Mt * 128) return;
  const __nv_bfloat16* src = rows[row];
  float amax = 0.f;
  if (src)
    for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(__bfloat162float(src[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sc = amax == 0.f ? 1.f : __fdiv_rn(amax, 127.f);
  if (lane == 0) scales[row] = sc;
  const int mt = row >> 7, r = row & 127;
  for (int c = lane; c < KB8 * 8; c += 32) {            // 16-element chunks along K
    const int kb = c >> 3, ch = c & 7, k0 = c * 16;
    uint32_t word[4] = {0, 0, 0, 0};
    if (src) {
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int k = k0 + q;
        const float v = k < K ? rintf(__fdiv_rn(__bfloat162float(src[k]), sc)) : 0.f;   // ties to even
        const int code = max(-127, min(127, (int)v));
        word[q >> 2] |= (uint32_t)(code & 0xFF) << ((q & 3) * 8);
      }
    }
    *reinterpret_cast<uint4*>(dst + ((size_t)mt * KB8 + kb) * kTileBytesPack + sw128_chunk_byte(r, ch)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// Group-wise symmetric int4 packing (W4A16): per row and group of 128 inputs, scale = max|w| / 7
// (1 for a zero group), code = round-to-nearest-even(w / scale) clamped to [-7, 7].  Tiles hold
// 128 rows x 256 codes (two per byte, low nibble first), 16-byte chunks of 32 codes swizzled;
// scales [row][ceil(K / 128)].  One warp per row.
__global__ void quant_int4_kernel(const __nv_bfloat16* const* __restrict__ rows, int K, int Mt, int KB4,
                                  uint8_t* __restrict__ dst, float* __restrict__ scales) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= Mt * 128) return;
  const __nv_bfloat16* src = rows[row];
  const int ng = (K + 127) / 128;
  for (int g = lane; g < ng; g += 32) {
    float amax = 0.f;
    if (src)
      for (int k = g * 128; k < min(K, g * 128 + 128); ++k) amax = fmaxf(amax, fabsf(__bfloat162float(src[k])));
    scales[(size_t)row * ng + g] = amax == 0.f ? 1.f : __fdiv_rn(amax, 7.f);
  }
  __syncwarp();
  const int mt = row >> 7, r = row & 127;
  for (int c = lane; c < KB4 * 8; c += 32) {            // 32-code chunks along K
    const int kb = c >> 3, ch = c & 7, k0 = c * 32;
    uint32_t word[4] = {0, 0, 0, 0};
    if (src && k0 < K) {   // (chunks past K keep zero codes)
      const float sc = scales[(size_t)row * ng + k0 / 128];   // written by this warp above
#pragma unroll 8
      for (int q = 0; q < 32; ++q) {
        const int k = k0 + q;
        const float v = k < K ? rintf(__fdiv_rn(__bfloat162float(src[k]), sc)) : 0.f;   // ties to even
        const int code = max(-7, min(7, (int)v));
        word[q >> 3] |= (uint32_t)(code & 0xF) << ((q & 7) * 4);
      }
    }
    *reinterpret_cast<uint4*>(dst + ((size_t)mt * KB4 + kb) * kTileBytesPack + sw128_chunk_byte(r, ch)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
}

// Prefix K/V producer operand of layer l: per prefix token row t = b * P + j, the sum of squares
// of h (one part) and the hi/lo bf16 tiles of h * gain, 8 inputs (one 16-byte chunk of each tile)
// per thread.  hidden [B][L][P][Hv] bf16, Hv % 8 == 0.  Launched chained after the previous
// layer's GEMM: the operand is overwritten only after that GEMM has finished reading it.
__global__ void prefix_operand_kernel(const __nv_bfloat16* __restrict__ hidden, const float* __restrict__ gain,
                                      int L, int l, int P, int Hv, float* ss, __nv_bfloat16* tiles, int NT, int KB) {
  pdl_trigger();
  const int t = blockIdx.x, b = t / P, j = t % P;
  const __nv_bfloat16* h = hidden + (((size_t)b * L + l) * P + j) * Hv;
  __shared__ float red[32];
  float acc = 0.f;
  uint4 raw[2];
  float4 g[4];
  const int nch = Hv / 8;
  // static inputs first, then wait for the previous kernel of the stream
  int c = threadIdx.x;
  const bool two = c + (int)blockDim.x < nch;
  if (c < nch) {
    raw[0] = __ldg(reinterpret_cast<const uint4*>(h) + c);
    g[0] = __ldg(reinterpret_cast<const float4*>(gain) + 2 * c);
    g[1] = __ldg(reinterpret_cast<const float4*>(gain) + 2 * c + 1);
  }
  if (two) {
    raw[1] = __ldg(reinterpret_cast<const uint4*>(h) + c + blockDim.x);
    g[2] = __ldg(reinterpret_cast<const float4*>(gain) + 2 * (c + blockDim.x));
    g[3] = __ldg(reinterpret_cast<const float4*>(gain) + 2 * (c + blockDim.x) + 1);
  }
  pdl_wait();
  for (int rep = 0; rep < 2 && c < nch; ++rep, c += blockDim.x) {
    const uint4 r = rep == 0 ? raw[0] : raw[1];
    const float gg[8] = {rep == 0 ? g[0].x : g[2].x, rep == 0 ? g[0].y : g[2].y, rep == 0 ? g[0].z : g[2].z,
                         rep == 0 ? g[0].w : g[2].w, rep == 0 ? g[1].x : g[3].x, rep == 0 ? g[1].y : g[3].y,
                         rep == 0 ? g[1].z : g[3].z, rep == 0 ? g[1].w : g[3].w};
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&w[q]);
      const float x0 = __low2float(pr), x1 = __high2float(pr);
      acc = fmaf(x0, x0, acc);
      acc = fmaf(x1, x1, acc);
      const float v0 = x0 * gg[2 * q], v1 = x1 * gg[2 * q + 1];
      const __nv_bfloat162 hi = __floats2bfloat162_rn(v0, v1);
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v0 - __low2float(hi), v1 - __high2float(hi));
      hw[q] = *reinterpret_cast<const uint32_t*>(&hi);
      lw[q] = *reinterpret_cast<const uint32_t*>(&lo);
    }
    const size_t off = operand_offset(t, c * 8, NT, KB);
    *reinterpret_cast<uint4*>(tiles + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(tiles + off + (size_t)NT * 64) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
  for (; c < nch; c += blockDim.x) {   // widths past 2 x blockDim x 8
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(h) + c);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&w[q]);
      const float x0 = __low2float(pr), x1 = __high2float(pr);
      acc = fmaf(x0, x0, acc);
      acc = fmaf(x1, x1, acc);
      const float v0 = x0 * __ldg(gain + c * 8 + 2 * q), v1 = x1 * __ldg(gain + c * 8 + 2 * q + 1);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(v0, v1);
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v0 - __low2float(hi), v1 - __high2float(hi));
      hw[q] = *reinterpret_cast<const uint32_t*>(&hi);
      lw[q] = *reinterpret_cast<const uint32_t*>(&lo);
    }
    const size_t off = operand_offset(t, c * 8, NT, KB);
    *reinterpret_cast<uint4*>(tiles + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(tiles + off + (size_t)NT * 64) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s2 = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s2 += red[w];
    ss[t] = s2;
  }
}

// prefix rows of one layer's caches -> fp32 k, v [B][P][nkv][hd]
__global__ void prefix_kv_readback_kernel(const __nv_bfloat16* kc, const __nv_bfloat16* vct, float* k, float* v, int B,
                                          int P, int nkv, int hd, int Lpad) {
  const size_t n = (size_t)B * P * nkv * hd;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const int d = e % hd, g = (e / hd) % nkv, j = (e / ((size_t)hd * nkv)) % P, b = e / ((size_t)hd * nkv * P);
    const size_t cache = (size_t)b * nkv + g;
    k[e] = __bfloat162float(kc[(cache * Lpad + j) * hd + d]);
    v[e] = __bfloat162float(vct[(cache * hd + d) * Lpad + j]);
  }
}

// ---------------------------------------------------------------- prefix layout (set_prefix)
// user K, V: [B][L][P][nkv][hd]  ->  K cache [L][B][nkv][Lpad][hd], V^T cache [L][B][nkv][hd][Lpad]
__global__ void prefix_layout_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                     __nv_bfloat16* kc, __nv_bfloat16* vct, int B, int L, int P, int nkv, int hd,
                                     int Lpad) {
  const size_t total = (size_t)B * L * P * nkv * hd;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int d = (int)(e % hd);
    size_t r = e / hd;
    const int g = (int)(r % nkv); r /= nkv;
    const int pp = (int)(r % P); r /= P;
    const int l = (int)(r % L);
    const int b = (int)(r / L);
    const size_t cache = (((size_t)l * B + b) * nkv + g);
    kc[(cache * Lpad + pp) * hd + d] = k[e];
    vct[(cache * hd + d) * Lpad + pp] = v[e];
  }
}

// ---------------------------------------------------------------- failure-detection probe
// Waits on an mbarrier that nothing arrives on, with a bounded number of attempts: the wait runs
// out, the kernel records DEV_ERR_TIMEOUT_MMA in the status word and returns normally.
__global__ void wait_probe_kernel(unsigned limit, unsigned* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, limit, status, DEV_ERR_TIMEOUT_MMA);
  __syncthreads();
}

// ---------------------------------------------------------------- debug read-outs
// ss[t] = sum_k h[t][k]^2 for one row per CTA (fixed-order block reduction), and the row's
// GEMM operand h (1 + scale) as hi/lo tiles
__global__ void row_operand_kernel(const float* h, float* ss, __nv_bfloat16* tiles, const float* scale, int H, int NT,
                                   int KB) {
  __shared__ float red[32];
  const int t = blockIdx.x, tid = threadIdx.x;
  float s = 0.f;
  for (int k = tid; k < H; k += blockDim.x) {
    const float v = h[(size_t)t * H + k];
    s = fmaf(v, v, s);
    store_operand(tiles, t, k, NT, KB, v * (1.f + scale[k]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((tid & 31) == 0) red[tid >> 5] = s;
  __syncthreads();
  if (tid == 0) {
    float a = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) a += red[w];
    ss[t] = a;
  }
}
// hi/lo operand tiles [Nt][KB][2][NT][64] -> fp32 [Ntok][K] (hi + lo)
__global__ void untile_kernel(const __nv_bfloat16* tiles, float* out, int Ntok, int K, int NT, int KB) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < Ntok * K; e += gridDim.x * blockDim.x) {
    const int t = e / K, k = e % K;
    const size_t off = operand_offset(t, k, NT, KB);
    out[e] = __bfloat162float(tiles[off]) + __bfloat162float(tiles[off + (size_t)NT * 64]);
  }
}

// W . shift for every packed row of one op of one layer and every step:
// out[k][pr] = sum_c W[pr][c] shift_k[c], with W read back from the packed tiles (8-bit formats:
// decoded code times the row scale, i.e. exactly the weights the GEMM multiplies).  One warp per row.
__global__ void cshift_kernel(const uint8_t* __restrict__ wt, const float* __restrict__ wscale, int rows, int KBt,
                              int K, int wq, int spr, const float* __restrict__ shift, size_t shift_step_stride, int steps,
                              float* out, size_t out_step_stride) {
  const int pr = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pr >= rows) return;
  const int mt = pr >> 7, r = pr & 127;
  for (int k = 0; k < steps; ++k) {
    double acc = 0.0;
    const float* sh = shift + (size_t)k * shift_step_stride;
    for (int c = lane; c < K; c += 32) {
      float w;
      if (wq == 3) {   // int4 code times its group's scale, rounded to bf16 as the GEMM widens it
        const uint8_t* tile = wt + ((size_t)mt * KBt + c / 256) * kTileBytesPack;
        const int kk = c % 256;
        const int nib = (tile[sw128_chunk_byte(r, kk / 32) + (kk % 32) / 2] >> (4 * (kk & 1))) & 0xF;
        w = __bfloat162float(__float2bfloat16_rn((float)((nib ^ 8) - 8) * wscale[(size_t)pr * spr + c / 128]));
      } else if (wq) {   // 8-bit codes (1: e4m3, 2: int8) times the row scale
        const uint8_t* tile = wt + ((size_t)mt * KBt + c / 128) * kTileBytesPack;
        const uint8_t code = tile[sw128_chunk_byte(r, (c % 128) / 16) + (c % 16)];
        const uint32_t pair = wq == 2 ? s8x2_to_bf16x2((uint16_t)code) : e4m3x2_to_bf16x2((uint16_t)code);
        w = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&pair)) * wscale[pr];
      } else {
        const __nv_bfloat16* tile = reinterpret_cast<const __nv_bfloat16*>(wt + ((size_t)mt * KBt + c / 64) * kTileBytesPack);
        w = __bfloat162float(tile[sw128_elem_offset(r, c % 64)]);
      }
      acc += (double)w * (double)sh[c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[(size_t)k * out_step_stride + pr] = (float)acc;
  }
}
__global__ void bf16_to_f32_kernel(const __nv_bfloat16* in, float* out, size_t n) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
    out[e] = __bfloat162float(in[e]);
}
// self rows of the layer caches -> fp32 k [Ntok][nkv][hd], v [Ntok][nkv][hd]
__global__ void self_kv_kernel(const __nv_bfloat16* kc, const __nv_bfloat16* vct, float* k, float* v, int B, int Ts,
                               int nkv, int hd, int P, int Lpad) {
  const int n = B * Ts * nkv * hd;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int d = e % hd, g = (e / hd) % nkv, t = e / (hd * nkv);
    const int b = t / Ts, j = t % Ts;
    const size_t cache = (size_t)b * nkv + g;
    k[e] = __bfloat162float(kc[(cache * Lpad + P + j) * hd + d]);
    v[e] = __bfloat162float(vct[(cache * hd + d) * Lpad + P + j]);
  }
}

// q of the attention layout [B][nkv][Rpad][hd] (rows head_in_group * Ts + token) -> fp32 [Ntok][nq][hd]
__global__ void q_trace_kernel(const __nv_bfloat16* qb, float* out, int B, int Ts, int nq, int nkv, int hd, int Rpad) {
  const int n = B * Ts * nq * hd, rep = nq / nkv;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int d = e % hd, head = (e / hd) % nq, t = e / (hd * nq);
    const int b = t / Ts, j = t % Ts, g = head / rep;
    out[e] = __bfloat162float(qb[(((size_t)b * nkv + g) * Rpad + (head % rep) * Ts + j) * hd + d]);
  }
}

}  // namespace vla
