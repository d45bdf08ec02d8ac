"""Seeded synthetic inputs for the action-expert denoise loop.

This module is shared by the CPU oracle and the GPU path.  It only draws
numbers and lays them out: it holds none of the method's arithmetic.

Workload shapes follow the five workloads the action expert is measured on:

* ``tiny``     -- 2-layer DiT, hidden 256, 4/2 heads of 64, SwiGLU 704,
                  16 action tokens x 7, 64 prefix tokens, 4 Euler steps.
* ``starvla``  -- StarVLA-shaped action head ("AI Infra如何优化VLA",
                  section 整体方案: 4 steps x 36-layer DiT, ~1B parameters):
                  hidden 1536, 12/4 heads of 128, SwiGLU 4096, 16 action
                  tokens + 1 state token, action_dim 7, 300 prefix tokens.
* ``pi05``     -- pi0.5-shaped expert (APXInf article, section on CUDA
                  Graph / FP8 / Rust: 10 flow steps): 18 layers, hidden
                  1024, 8/1 heads of 256, SwiGLU 4096, 50 action tokens x
                  32, 800 prefix tokens.
* ``pi05_fp8`` -- ``pi05`` with e4m3 linear weights (per-output-channel
                  fp32 scales), 1 or 10 steps.
* ``pi05_int8`` -- ``pi05`` with int8 linear weights (per-output-channel
                  fp32 scales; the INT8 fallback of the same article).
* ``pi05_int4`` -- ``pi05`` with int4 linear weights (W4A16, fp32 scales per
                  output channel and 128 inputs).
* batch sweep  -- ``tiny`` and ``starvla`` at batch 1, 4, 16 and 64.

Random numbers: numpy's PCG64 bit generator (O'Neill, "PCG: A Family of
Simple Fast Space-Efficient Statistically Good Algorithms for Random Number
Generation", 2014) under a ``SeedSequence``.  Weight matrix number ``i`` in
canonical order comes from its own stream ``[seed, 0, i]`` (so matrices can be
drawn in parallel); the per-sample inputs of sample ``b`` come from the stream
``[seed, 1, b]``, so a sample's inputs do not depend on the batch it sits in.
Weights are N(0, 0.02); noise, state and prefix K/V are N(0, 1); all of them
are drawn in fp32 and rounded to bf16 (round to nearest even), which is how
the workloads specify their inputs.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np

__all__ = [
    "Dims", "CONFIGS", "config", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "generate_weights", "generate_sample", "generate_inputs", "WEIGHT_ORDER",
    "LAYER_WEIGHT_ORDER", "weight_shapes", "abi_dims", "BATCH_SWEEP",
]


@dataclasses.dataclass(frozen=True)
class Dims:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    inter: int
    t_emb_dim: int
    action_dim: int
    n_action_tokens: int
    has_state_token: int
    n_prefix: int
    steps: int
    batch: int = 1
    wtype: str = "bf16"          # "bf16", "fp8_e4m3", "int8" or "int4_g128"
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def qd(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kd(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def ts(self) -> int:
        """Self tokens per sample: action tokens plus the optional state token."""
        return self.n_action_tokens + self.has_state_token

    def replace(self, **kw) -> "Dims":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, Dims] = {
    "tiny": Dims(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                 inter=704, t_emb_dim=256, action_dim=7, n_action_tokens=16,
                 has_state_token=0, n_prefix=64, steps=4),
    "starvla": Dims(n_layers=36, hidden=1536, n_q_heads=12, n_kv_heads=4, head_dim=128,
                    inter=4096, t_emb_dim=256, action_dim=7, n_action_tokens=16,
                    has_state_token=1, n_prefix=300, steps=4),
    "pi05": Dims(n_layers=18, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=256,
                 inter=4096, t_emb_dim=256, action_dim=32, n_action_tokens=50,
                 has_state_token=0, n_prefix=800, steps=10),
    "pi05_fp8": Dims(n_layers=18, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=256,
                     inter=4096, t_emb_dim=256, action_dim=32, n_action_tokens=50,
                     has_state_token=0, n_prefix=800, steps=10, wtype="fp8_e4m3"),
    "pi05_int8": Dims(n_layers=18, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=256,
                      inter=4096, t_emb_dim=256, action_dim=32, n_action_tokens=50,
                      has_state_token=0, n_prefix=800, steps=10, wtype="int8"),
    "pi05_int4": Dims(n_layers=18, hidden=1024, n_q_heads=8, n_kv_heads=1, head_dim=256,
                      inter=4096, t_emb_dim=256, action_dim=32, n_action_tokens=50,
                      has_state_token=0, n_prefix=800, steps=10, wtype="int4_g128"),
}

BATCH_SWEEP = (1, 4, 16, 64)


def config(name: str, **overrides) -> Dims:
    return CONFIGS[name].replace(**overrides) if overrides else CONFIGS[name]


# ---------------------------------------------------------------- bf16 bits

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 bit patterns.

    Inputs are finite (drawn from a normal distribution), so no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- weights

LAYER_WEIGHT_ORDER = ("w_ada", "b_ada", "wq", "wk", "wv", "wo", "wg", "wu", "wd")
WEIGHT_ORDER = ("w_in", "b_in", "w_state", "b_state", "layers", "w_fada", "b_fada",
                "w_out", "b_out")


def weight_shapes(d: Dims) -> Dict[str, tuple]:
    H, A, Dt, I = d.hidden, d.action_dim, d.t_emb_dim, d.inter
    return {
        "w_in": (H, A), "b_in": (H,), "w_state": (H, A), "b_state": (H,),
        "w_ada": (6 * H, Dt), "b_ada": (6 * H,),
        "wq": (d.qd, H), "wk": (d.kd, H), "wv": (d.kd, H), "wo": (H, d.qd),
        "wg": (I, H), "wu": (I, H), "wd": (H, I),
        "w_fada": (2 * H, Dt), "b_fada": (2 * H,),
        "w_out": (A, H), "b_out": (A,),
    }


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    chunk = 1 << 24
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        z = rng.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            z *= np.float32(std)
        out[s:e] = f32_to_bf16_bits(z)
    return out.reshape(shape)


def _weight_list(d: Dims):
    """(key, layer or None, shape) in canonical draw order."""
    sh = weight_shapes(d)
    items = [("w_in", None), ("b_in", None)]
    if d.has_state_token:
        items += [("w_state", None), ("b_state", None)]
    for l in range(d.n_layers):
        items += [(name, l) for name in LAYER_WEIGHT_ORDER]
    items += [(name, None) for name in ("w_fada", "b_fada", "w_out", "b_out")]
    return [(k, l, sh[k]) for k, l in items]


def generate_weights(d: Dims, seed: int = 0, std: float = 0.02, threads: int = 8) -> Dict[str, object]:
    """All weights as bf16 bit patterns (uint16), each matrix from its own seeded stream.

    Canonical order: in-proj (W, b), state-proj (W, b; only when a state token exists), then
    per layer adaLN (W, b), q, k, v, o, gate, up, down, then the final adaLN (W, b) and the
    out-proj (W, b).  Matrices are ``[out, in]`` row-major.
    """
    from concurrent.futures import ThreadPoolExecutor

    items = _weight_list(d)

    def draw(i):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0, i])))
        return _normal_bf16(rng, items[i][2], std)

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        arrays = list(ex.map(draw, range(len(items))))
    w: Dict[str, object] = {"layers": [dict() for _ in range(d.n_layers)]}
    for (key, layer, _), a in zip(items, arrays):
        if layer is None:
            w[key] = a
        else:
            w["layers"][layer][key] = a
    return w


def generate_sample(d: Dims, b: int, seed: int = 0, n_prefix: int | None = None) -> Dict[str, np.ndarray]:
    """Inputs of sample ``b``: noise [T, A], state [A] (if any), prefix K and V [L, P, nkv, hd]."""
    P = d.n_prefix if n_prefix is None else n_prefix
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1, b])))
    s: Dict[str, np.ndarray] = {}
    s["noise"] = _normal_bf16(rng, (d.n_action_tokens, d.action_dim), 1.0)
    if d.has_state_token:
        s["state"] = _normal_bf16(rng, (d.action_dim,), 1.0)
    k = np.empty((d.n_layers, P, d.n_kv_heads, d.head_dim), dtype=np.uint16)
    v = np.empty_like(k)
    for l in range(d.n_layers):
        k[l] = _normal_bf16(rng, (P, d.n_kv_heads, d.head_dim), 1.0)
        v[l] = _normal_bf16(rng, (P, d.n_kv_heads, d.head_dim), 1.0)
    s["k"] = k
    s["v"] = v
    return s


def generate_inputs(d: Dims, seed: int = 0, n_prefix: int | None = None) -> Dict[str, np.ndarray]:
    """Batched per-sample inputs: noise [B, T, A], state [B, A], K/V [B, L, P, nkv, hd]."""
    samples = [generate_sample(d, b, seed, n_prefix) for b in range(d.batch)]
    out = {key: np.stack([s[key] for s in samples]) for key in samples[0]}
    return out


def abi_dims(d: Dims, max_prefix: int | None = None) -> Dict[str, object]:
    """The ``vla_ae_dims`` fields for a workload (field renaming only)."""
    return dict(n_layers=d.n_layers, hidden=d.hidden, n_q_heads=d.n_q_heads, n_kv_heads=d.n_kv_heads,
                head_dim=d.head_dim, inter=d.inter, t_emb_dim=d.t_emb_dim, action_dim=d.action_dim,
                n_action_tokens=d.n_action_tokens, has_state_token=d.has_state_token,
                max_prefix=d.n_prefix if max_prefix is None else max_prefix, batch=d.batch,
                rope_theta=d.rope_theta, rms_eps=d.rms_eps, wtype={"bf16": 0, "fp8_e4m3": 1, "int8": 2, "int4_g128": 3}[d.wtype])
