"""What the action-expert denoise loop computes, in plain float64 numpy (test infrastructure only).

Sources and readings:

* Flow-matching Euler from noise over N fixed steps, x <- x + dt * v: "AI Infra如何优化VLA"
  (RimBot), section 整体方案 (4 steps x 36-layer DiT action head); the APXInf article,
  section "CUDA Graph、FP8 和 Rust" (10 steps, and a 1-step variant).  Reading: t runs
  from 1 (noise) to 0 with signed dt = -1/N and t_k = 1 - k/N.
* RMSNorm as an fp32 row operation (mean of squares, rsqrt, scale): RimBot page, section
  算子开发.  Reading: eps = 1e-6 and no learned weight (adaLN supplies the scale).
* Half-split RoPE ("分半旋转") on Q and K: RimBot page, section 算子开发.  Reading: base
  10000; self tokens sit at positions P..P+Ts-1; the cached prefix K is already rotated.
* Sin/Cos time embedding: RimBot page, section 整体方案 (operator list).  Reading:
  [cos | sin] of 1000 * t * 10000^(-i/half), then SiLU, then per-layer adaLN-Zero:
  shift/scale/gate for attention and MLP (6H), and a final shift/scale (2H).
* GQA attention of the action tokens over themselves and the cached VLM prefix, no mask;
  consecutive q heads share a kv head.  SwiGLU MLP (SiLU(gate) * up -> down).  Fused QKV
  and SwiGLU are named in the RimBot page, section 算子融合.
* Biases only on adaLN, in-proj, state-proj and out-proj.
"""

from __future__ import annotations

import math
from typing import Callable, Dict, List, Optional

import numpy as np

from .fp8 import quantize_rowwise_e4m3, dequantize_rowwise_e4m3
from .int8 import quantize_rowwise_int8, dequantize_rowwise_int8
from .int4 import quantize_groupwise_int4, dequantize_groupwise_int4


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact widening)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ sampler

def t_schedule(n_steps: int):
    """t_k = 1 - k/N for k = 0..N-1 and the signed step dt = -1/N."""
    if n_steps < 1:
        raise ValueError("n_steps must be >= 1")
    return [1.0 - k / n_steps for k in range(n_steps)], -1.0 / n_steps


def check_t_grid(t_grid) -> List[float]:
    """A time grid t_0 > t_1 > ... > t_n (n >= 1, finite values) as floats.

    Step skipping ("跨XPU平台表征视觉-语言-动作模型" sections 5.2 and 5.3.2: DP-Cache drops a fixed set
    of intermediate diffusion steps) and the one-step variant (APXInf article, section "CUDA
    Graph、FP8 和 Rust") are such grids: a dropped step's interval joins the step before it, which
    for Euler is the same as reusing that step's velocity over the dropped interval."""
    g = [float(t) for t in t_grid]
    if len(g) < 2:
        raise ValueError("a time grid needs at least two points")
    if not all(math.isfinite(t) for t in g):
        raise ValueError("time grid values must be finite")
    if not all(b < a for a, b in zip(g, g[1:])):
        raise ValueError("time grid must be strictly decreasing")
    return g


def uniform_grid(n_steps: int) -> List[float]:
    """t_k = 1 - k/N for k = 0..N (t_N = 0): the grid of the fixed-step loop."""
    if n_steps < 1:
        raise ValueError("n_steps must be >= 1")
    return [1.0 - k / n_steps for k in range(n_steps + 1)]


def euler_integrate_grid(x0: np.ndarray, t_grid, v_fn: Callable[[np.ndarray, float], np.ndarray]) -> np.ndarray:
    """Explicit Euler along a time grid: x_{k+1} = x_k + (t_{k+1} - t_k) * v(x_k, t_k)."""
    g = check_t_grid(t_grid)
    x = np.array(x0, dtype=np.float64, copy=True)
    for t0, t1 in zip(g, g[1:]):
        x = x + (t1 - t0) * v_fn(x, t0)
    return x


def euler_integrate_switch(x0: np.ndarray, n_steps: int, n_stale: int,
                           v_before: Callable[[np.ndarray, float], np.ndarray],
                           v_after: Callable[[np.ndarray, float], np.ndarray]) -> np.ndarray:
    """Fixed-step Euler whose field changes after ``n_stale`` steps ("跨XPU平台表征视觉-语言-动作模型"
    section 5.3, V-AEFusion: the first steps reuse the previous cycle's visual features):
    x_{k+1} = x_k + dt * v_before(x_k, t_k) for k < n_stale, then v_after."""
    if not 0 <= n_stale <= n_steps:
        raise ValueError("0 <= n_stale <= n_steps")
    ts, dt = t_schedule(n_steps)
    x = np.array(x0, dtype=np.float64, copy=True)
    for k, t in enumerate(ts):
        x = x + dt * (v_before if k < n_stale else v_after)(x, t)
    return x


def euler_integrate(x0: np.ndarray, n_steps: int, v_fn: Callable[[np.ndarray, float], np.ndarray]) -> np.ndarray:
    """Fixed-step explicit Euler from t = 1 to t = 0: x_{k+1} = x_k + dt * v(x_k, t_k)."""
    ts, dt = t_schedule(n_steps)
    x = np.array(x0, dtype=np.float64, copy=True)
    for t in ts:
        x = x + dt * v_fn(x, t)
    return x


# ------------------------------------------------------------------ elementwise pieces

def timestep_embedding(t: float, dim: int = 256, max_period: float = 10000.0,
                       scale: float = 1000.0) -> np.ndarray:
    """[cos(a_0..a_{half-1}), sin(a_0..a_{half-1})] with a_i = scale * t * max_period^(-i/half)."""
    half = dim // 2
    i = np.arange(half, dtype=np.float64)
    freqs = np.exp(-math.log(max_period) * i / half)
    a = scale * t * freqs
    return np.concatenate([np.cos(a), np.sin(a)])


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def rms_norm(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """h / sqrt(mean(h^2) + eps) over the last axis."""
    ms = np.mean(h * h, axis=-1, keepdims=True)
    return h / np.sqrt(ms + eps)


def modulate(u: np.ndarray, shift: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return u * (1.0 + scale) + shift


def rope_positions_angles(pos: np.ndarray, head_dim: int, theta: float = 10000.0) -> np.ndarray:
    """theta_{p,i} = p * theta^(-2i/hd) for i < hd/2; shape [len(pos), hd/2]."""
    half = head_dim // 2
    i = np.arange(half, dtype=np.float64)
    inv = theta ** (-2.0 * i / head_dim)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]


def rope_half(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """Half-split rotation of every head vector: x is [T, n_heads, hd], pos is [T].

    (x_i, x_{i+hd/2}) -> (x_i cos - x_{i+hd/2} sin, x_{i+hd/2} cos + x_i sin).
    """
    hd = x.shape[-1]
    half = hd // 2
    ang = rope_positions_angles(pos, hd, theta)[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q_h k_g^T / sqrt(hd)) v_g for every q head h, g = h // (nq / nkv); no mask.

    q is [T, nq, hd]; k and v are [Lk, nkv, hd]; returns [T, nq, hd].
    """
    T, nq, hd = q.shape
    nkv = k.shape[1]
    rep = nq // nkv
    out = np.empty((T, nq, hd), dtype=np.float64)
    if k.shape[0] == 0:
        raise ValueError("attention over an empty key set")
    for h in range(nq):
        g = h // rep
        s = q[:, h, :] @ k[:, g, :].T / math.sqrt(hd)          # [T, Lk]
        s = s - np.max(s, axis=1, keepdims=True)
        p = np.exp(s)
        p = p / np.sum(p, axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def linear(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray] = None) -> np.ndarray:
    """y = x W^T (+ b) with W stored [out, in]."""
    y = x @ w.T
    return y if b is None else y + b


def swiglu(x: np.ndarray, wg: np.ndarray, wu: np.ndarray) -> np.ndarray:
    return silu(linear(x, wg)) * linear(x, wu)


def prefix_kv(h: np.ndarray, wk: np.ndarray, wv: np.ndarray, gain: np.ndarray, n_kv_heads: int,
              eps: float = 1e-6, theta: float = 10000.0):
    """The VLM side of the cached prefix for one layer ("AI Infra如何优化VLA", section 算子开发: the
    RMSNorm, K/V projection and RoPE of the prefill).  h [P, Hv] are the layer's input hidden
    states of the P prefix tokens; x = rms_norm(h) * gain; K = rope_half(x Wk^T) at positions
    0..P-1, V = x Wv^T; returns K, V as [P, n_kv_heads, hd]."""
    x = rms_norm(h, eps) * gain
    P = h.shape[0]
    k = linear(x, wk).reshape(P, n_kv_heads, -1)
    v = linear(x, wv).reshape(P, n_kv_heads, -1)
    return rope_half(k, np.arange(P, dtype=np.float64), theta), v


# ------------------------------------------------------------------ weights

_LAYER_LINEARS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")


class OracleWeights:
    """float64 view of the synthetic bf16 weights (optionally with dequantised 8-bit linears).

    ``quantized`` = ``"fp8_e4m3"`` (or ``True``) replaces each per-layer q/k/v/o/gate/up/down
    weight W by W' = e4m3(W / s) * s, ``"int8"`` by W' = round(W / s) * s (one scale per output
    channel), ``"int4_g128"`` by W' = bf16(round(W / s) * s) (one scale per output channel and
    128 inputs); adaLN, in/out/state projections stay bf16.  ``False`` / ``"bf16"``: none.
    """

    def __init__(self, w: Dict[str, object], d, quantized=False):
        self.d = d
        if quantized is True:
            quantized = "fp8_e4m3"
        self.quantized = False if quantized in (False, None, "bf16") else quantized
        if self.quantized not in (False, "fp8_e4m3", "int8", "int4_g128"):
            raise ValueError(f"unknown weight format {quantized!r}")
        self._raw = w
        self.top = {k: bf16_to_f64(v) for k, v in w.items() if k != "layers"}
        self._cache: Dict[int, Dict[str, np.ndarray]] = {}

    def layer(self, l: int) -> Dict[str, np.ndarray]:
        if l in self._cache:
            return self._cache[l]
        raw = self._raw["layers"][l]
        lw = {k: bf16_to_f64(v) for k, v in raw.items()}
        if self.quantized == "fp8_e4m3":
            for k in _LAYER_LINEARS:
                codes, scales = quantize_rowwise_e4m3(lw[k].astype(np.float32))
                lw[k] = dequantize_rowwise_e4m3(codes, scales)
        elif self.quantized == "int8":
            for k in _LAYER_LINEARS:
                codes, scales = quantize_rowwise_int8(lw[k].astype(np.float32))
                lw[k] = dequantize_rowwise_int8(codes, scales)
        elif self.quantized == "int4_g128":
            for k in _LAYER_LINEARS:
                codes, scales = quantize_groupwise_int4(lw[k].astype(np.float32))
                lw[k] = dequantize_groupwise_int4(codes, scales)
        self._cache[l] = lw
        return lw


def adaln_table(w_ada: np.ndarray, b_ada: np.ndarray, t: float, t_emb_dim: int) -> np.ndarray:
    """W_ada SiLU(temb(t)) + b_ada."""
    c = silu(timestep_embedding(t, t_emb_dim))
    return w_ada @ c + b_ada


# ------------------------------------------------------------------ the velocity net

def dit_layer(h: np.ndarray, lw: Dict[str, np.ndarray], mod: np.ndarray, k_prefix: np.ndarray,
              v_prefix: np.ndarray, pos: np.ndarray, d, trace: Optional[Dict[str, np.ndarray]] = None) -> np.ndarray:
    """One DiT layer on the self tokens h [Ts, H].

    mod = [shift_a, scale_a, gate_a, shift_m, scale_m, gate_m] (each H).
    k_prefix / v_prefix are [P, nkv, hd].  ``trace`` (if given) receives the intermediates.
    """
    H = d.hidden
    sh_a, sc_a, g_a, sh_m, sc_m, g_m = (mod[i * H:(i + 1) * H] for i in range(6))
    Ts = h.shape[0]
    u = modulate(rms_norm(h, d.rms_eps), sh_a, sc_a)
    q = linear(u, lw["wq"]).reshape(Ts, d.n_q_heads, d.head_dim)
    k = linear(u, lw["wk"]).reshape(Ts, d.n_kv_heads, d.head_dim)
    v = linear(u, lw["wv"]).reshape(Ts, d.n_kv_heads, d.head_dim)
    q = rope_half(q, pos, d.rope_theta)
    k = rope_half(k, pos, d.rope_theta)
    k_all = np.concatenate([k_prefix, k], axis=0)
    v_all = np.concatenate([v_prefix, v], axis=0)
    o = gqa_attention(q, k_all, v_all).reshape(Ts, d.qd)
    h1 = h + g_a * linear(o, lw["wo"])
    u2 = modulate(rms_norm(h1, d.rms_eps), sh_m, sc_m)
    m = swiglu(u2, lw["wg"], lw["wu"])
    h2 = h1 + g_m * linear(m, lw["wd"])
    if trace is not None:
        trace.update(u=u, q=q, k=k, v=v, o=o, h_attn=h1, u2=u2, m=m, h_out=h2)
    return h2


def embed_tokens(x: np.ndarray, state: Optional[np.ndarray], W: OracleWeights, d) -> np.ndarray:
    """Self-token sequence: [W_st s + b_st] (when a state token exists), then W_in x_j + b_in."""
    top = W.top
    rows = []
    if d.has_state_token:
        rows.append(linear(state[None, :], top["w_state"], top["b_state"]))
    rows.append(linear(x, top["w_in"], top["b_in"]))
    return np.concatenate(rows, axis=0)


def velocity(x: np.ndarray, t: float, state: Optional[np.ndarray], W: OracleWeights,
             k_prefix: np.ndarray, v_prefix: np.ndarray, d,
             layer_trace: Optional[List[Dict[str, np.ndarray]]] = None) -> np.ndarray:
    """v_theta(x, t, prefix) for one sample: x [T, A]; k/v_prefix [L, P, nkv, hd]."""
    P = k_prefix.shape[1]
    h = embed_tokens(x, state, W, d)
    pos = P + np.arange(h.shape[0], dtype=np.float64)
    for l in range(d.n_layers):
        lw = W.layer(l)
        mod = adaln_table(lw["w_ada"], lw["b_ada"], t, d.t_emb_dim)
        tr = {} if layer_trace is not None else None
        if tr is not None:
            tr["h_in"] = h
        h = dit_layer(h, lw, mod, k_prefix[l], v_prefix[l], pos, d, tr)
        if layer_trace is not None:
            layer_trace.append(tr)
    fmod = adaln_table(W.top["w_fada"], W.top["b_fada"], t, d.t_emb_dim)
    sh_f, sc_f = fmod[:d.hidden], fmod[d.hidden:]
    u = modulate(rms_norm(h, d.rms_eps), sh_f, sc_f)
    act = u[d.has_state_token:]
    return linear(act, W.top["w_out"], W.top["b_out"])


def denoise(noise: np.ndarray, state: Optional[np.ndarray], W: OracleWeights, k_prefix: np.ndarray,
            v_prefix: np.ndarray, d, n_steps: int, t_grid=None) -> np.ndarray:
    """x_N of the N-step Euler loop for one sample (inputs already float64); with `t_grid`, the
    Euler loop along that time grid instead (n_steps is then ignored)."""
    v_fn = lambda x, t: velocity(x, t, state, W, k_prefix, v_prefix, d)
    if t_grid is not None:
        return euler_integrate_grid(noise, t_grid, v_fn)
    return euler_integrate(noise, n_steps, v_fn)


def denoise_stale(noise: np.ndarray, before, after, W: OracleWeights, d, n_steps: int, n_stale: int) -> np.ndarray:
    """x_N of the N-step loop whose first ``n_stale`` steps see prefix ``before`` and the rest
    ``after``; each prefix is (state, k_prefix, v_prefix) in float64 (state None without a state
    token)."""
    vb = lambda x, t: velocity(x, t, before[0], W, before[1], before[2], d)
    va = lambda x, t: velocity(x, t, after[0], W, after[1], after[2], d)
    return euler_integrate_switch(noise, n_steps, n_stale, vb, va)


def denoise_batch(weights_bits: Dict[str, object], inputs_bits: Dict[str, np.ndarray], d,
                  n_steps: Optional[int] = None, samples: Optional[List[int]] = None,
                  W: Optional[OracleWeights] = None, t_grid=None) -> np.ndarray:
    """Run ``denoise`` per sample on the synthetic bf16 inputs; returns [len(samples), T, A]."""
    n_steps = d.steps if n_steps is None else n_steps
    if W is None:
        W = OracleWeights(weights_bits, d, quantized=d.wtype)
    B = inputs_bits["noise"].shape[0]
    samples = list(range(B)) if samples is None else samples
    outs = []
    for b in samples:
        noise = bf16_to_f64(inputs_bits["noise"][b])
        state = bf16_to_f64(inputs_bits["state"][b]) if d.has_state_token else None
        kp = bf16_to_f64(inputs_bits["k"][b])
        vp = bf16_to_f64(inputs_bits["v"][b])
        outs.append(denoise(noise, state, W, kp, vp, d, n_steps, t_grid=t_grid))
    return np.stack(outs)
