"""Python binding of the B200 flow-matching action-expert library (``include/vla_ae.h``).

Argument marshalling only: every step of the denoise loop runs in the CUDA kernels of
``libvla_ae.so``.  There is no fallback: importing fails loudly when the library is missing.
The functions keep the C names; ``ActionExpert`` is a small convenience owner of one handle.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

from .build import LIB_PATH

__all__ = [
    "lib", "VlaAeDims", "VlaAeWeights", "VlaAeTrace", "VlaAeError", "ActionExpert",
    "vla_ae_create", "vla_ae_set_prefix", "vla_ae_denoise", "vla_ae_denoise_host", "vla_ae_status",
    "vla_ae_strerror", "vla_ae_destroy", "vla_ae_query", "vla_ae_debug_layer", "vla_ae_debug_velocity",
    "vla_ae_debug_weight", "vla_ae_bench_op", "vla_ae_set_prefix_static", "vla_ae_debug_wait_probe", "vla_ae_set_engine", "vla_ae_denoise_sched", "vla_ae_set_prefix_next", "vla_ae_denoise_stale", "vla_ae_attach_vlm_kv", "vla_ae_set_prefix_hidden",
    "vla_ae_debug_prefix_kv", "VlaAeVlmKvWeights", "BF16", "FP8_E4M3", "INT8", "INT4_G128", "Q_KERNELS_PER_LOOP", "Q_WEIGHT_BYTES", "Q_KV_BYTES",
    "Q_DEVICE_BYTES", "Q_SPLITS", "Q_OP_BYTES", "Q_ENGINE", "ENGINE_PER_OP", "ENGINE_PERSISTENT", "ENGINE_AUTO",
]

BF16, FP8_E4M3, INT8, INT4_G128 = 0, 1, 2, 3
Q_KERNELS_PER_LOOP, Q_WEIGHT_BYTES, Q_KV_BYTES, Q_DEVICE_BYTES, Q_SPLITS, Q_OP_BYTES, Q_ENGINE = 1, 2, 3, 4, 5, 6, 7
ENGINE_PER_OP, ENGINE_PERSISTENT, ENGINE_AUTO = 0, 1, 2
OK, EINVAL, ENOMEM, ECUDA, ENOPREFIX, ETIMEOUT, EUNSUPPORTED = 0, -1, -2, -3, -4, -5, -6

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: run flow_matching_action_euler_b200.build.build_library() "
                      "(or __graft_entry__.build()) first; there is no fallback path")
lib = ctypes.CDLL(LIB_PATH)


class VlaAeDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "inter", "t_emb_dim", "action_dim",
        "n_action_tokens", "has_state_token", "max_prefix", "batch")] + [
        ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("wtype", ctypes.c_int)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)


class VlaAeWeights(ctypes.Structure):
    _fields_ = [("w_in", _P), ("b_in", _P), ("w_state", _P), ("b_state", _P),
                ("w_ada", _PP), ("b_ada", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
                ("wg", _PP), ("wu", _PP), ("wd", _PP),
                ("w_fada", _P), ("b_fada", _P), ("w_out", _P), ("b_out", _P), ("on_device", ctypes.c_int)]


class VlaAeVlmKvWeights(ctypes.Structure):
    _fields_ = [("hidden_vlm", ctypes.c_int), ("rms_eps", ctypes.c_float), ("on_device", ctypes.c_int),
                ("wk", _PP), ("wv", _PP), ("gain", _PP)]


class VlaAeTrace(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("q", "k", "v", "o", "h_attn", "m")]


_H = ctypes.c_void_p


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


vla_ae_create = _sig("vla_ae_create", ctypes.c_int, ctypes.POINTER(VlaAeDims), ctypes.POINTER(VlaAeWeights),
                     ctypes.POINTER(_H))
vla_ae_set_prefix = _sig("vla_ae_set_prefix", ctypes.c_int, _H, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P)
vla_ae_denoise = _sig("vla_ae_denoise", ctypes.c_int, _H, _P, ctypes.c_int, _P, _P)
vla_ae_denoise_host = _sig("vla_ae_denoise_host", ctypes.c_int, _H, _P, ctypes.c_int, _P, _P)
vla_ae_status = _sig("vla_ae_status", ctypes.c_int, _H)
vla_ae_strerror = _sig("vla_ae_strerror", ctypes.c_char_p, ctypes.c_int)
vla_ae_destroy = _sig("vla_ae_destroy", None, _H)
vla_ae_query = _sig("vla_ae_query", ctypes.c_int, _H, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_longlong))
vla_ae_debug_layer = _sig("vla_ae_debug_layer", ctypes.c_int, _H, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P,
                          ctypes.POINTER(VlaAeTrace))
vla_ae_debug_velocity = _sig("vla_ae_debug_velocity", ctypes.c_int, _H, ctypes.c_int, ctypes.c_int, _P, _P)
vla_ae_debug_weight = _sig("vla_ae_debug_weight", ctypes.c_int, _H, ctypes.c_int, ctypes.c_int, _P, _P)
vla_ae_bench_op = _sig("vla_ae_bench_op", ctypes.c_int, _H, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P)
vla_ae_debug_wait_probe = _sig("vla_ae_debug_wait_probe", ctypes.c_int, _H, ctypes.c_uint)
vla_ae_set_engine = _sig("vla_ae_set_engine", ctypes.c_int, _H, ctypes.c_int)
vla_ae_attach_vlm_kv = _sig("vla_ae_attach_vlm_kv", ctypes.c_int, _H, ctypes.POINTER(VlaAeVlmKvWeights))
vla_ae_set_prefix_hidden = _sig("vla_ae_set_prefix_hidden", ctypes.c_int, _H, _P, ctypes.c_int, _P, _P)
vla_ae_debug_prefix_kv = _sig("vla_ae_debug_prefix_kv", ctypes.c_int, _H, ctypes.c_int, _P, _P)
vla_ae_set_prefix_next = _sig("vla_ae_set_prefix_next", ctypes.c_int, _H, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P)
vla_ae_denoise_stale = _sig("vla_ae_denoise_stale", ctypes.c_int, _H, _P, ctypes.c_int, ctypes.c_int, _P, _P)
vla_ae_denoise_sched = _sig("vla_ae_denoise_sched", ctypes.c_int, _H, _P, ctypes.POINTER(ctypes.c_float),
                            ctypes.c_int, _P, _P)
vla_ae_set_prefix_static = _sig("vla_ae_set_prefix_static", ctypes.c_int, _H, _P, _P, ctypes.c_int, _P, _P)


class VlaAeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {vla_ae_strerror(code).decode()} ({code})")
        self.code = code


def _check(code: int, what: str):
    if code != OK:
        raise VlaAeError(code, what)


def _ptr(a) -> Optional[int]:
    """Address of a numpy array or torch tensor (None stays NULL)."""
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    return a.ctypes.data


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        return None
    return getattr(stream, "cuda_stream", stream)


class ActionExpert:
    """Owns one ``vla_ae_t``.  ``dims`` is a mapping of the ``vla_ae_dims`` fields; ``weights`` a
    mapping with the ``vla_ae_weights`` names ("layers": list of per-layer dicts with w_ada, b_ada,
    wq, wk, wv, wo, wg, wu, wd), each a bf16 bit-pattern array (numpy uint16 on the host, or a
    torch CUDA tensor when ``on_device``)."""

    def __init__(self, dims: Dict[str, object], weights: Dict[str, object], on_device: bool = False):
        d = VlaAeDims()
        for name, _ in VlaAeDims._fields_:
            if name == "wtype":
                d.wtype = int(dims.get("wtype", BF16))
            elif name == "rope_theta":
                d.rope_theta = float(dims.get("rope_theta", 10000.0))
            elif name == "rms_eps":
                d.rms_eps = float(dims.get("rms_eps", 1e-6))
            else:
                setattr(d, name, int(dims[name]))
        self.dims = d
        layers = weights["layers"]
        self._keep = []

        def arr(key):
            ptrs = (ctypes.c_void_p * len(layers))(*[_ptr(lw[key]) for lw in layers])
            self._keep.append(ptrs)
            return ctypes.cast(ptrs, _PP)

        w = VlaAeWeights()
        for key in ("w_in", "b_in", "w_state", "b_state", "w_fada", "b_fada", "w_out", "b_out"):
            setattr(w, key, _ptr(weights.get(key)))
        for key in ("w_ada", "b_ada", "wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            setattr(w, key, arr(key))
        w.on_device = int(on_device)
        h = _H()
        _check(vla_ae_create(ctypes.byref(d), ctypes.byref(w), ctypes.byref(h)), "vla_ae_create")
        self.handle = h
        self._keep = []

    def set_prefix(self, k, v, n_prefix: int, state=None, on_device: bool = False, stream=None):
        _check(vla_ae_set_prefix(self.handle, _ptr(k), _ptr(v), int(n_prefix), _ptr(state), int(on_device),
                                 _stream_ptr(stream)), "vla_ae_set_prefix")

    def set_prefix_static(self, k_host, v_host, n_prefix: int, state_host=None, stream=None):
        """Allocation-free prefix upload from host buffers (see vla_ae_set_prefix_static)."""
        _check(vla_ae_set_prefix_static(self.handle, _ptr(k_host), _ptr(v_host), int(n_prefix), _ptr(state_host),
                                        _stream_ptr(stream)), "vla_ae_set_prefix_static")

    def denoise(self, noise, steps: int, out, stream=None):
        _check(vla_ae_denoise(self.handle, _ptr(noise), int(steps), _ptr(out), _stream_ptr(stream)),
               "vla_ae_denoise")

    def attach_vlm_kv(self, wk: Sequence, wv: Sequence, gain: Sequence, hidden_vlm: int, rms_eps: float = 1e-6):
        """Backbone K/V projections per layer (host bf16 arrays; see vla_ae_attach_vlm_kv)."""
        arr = lambda xs: (ctypes.c_void_p * len(xs))(*[_ptr(x) for x in xs])
        keep = (arr(wk), arr(wv), arr(gain))
        w = VlaAeVlmKvWeights(int(hidden_vlm), float(rms_eps), 0,
                              ctypes.cast(keep[0], _PP), ctypes.cast(keep[1], _PP), ctypes.cast(keep[2], _PP))
        _check(vla_ae_attach_vlm_kv(self.handle, ctypes.byref(w)), "vla_ae_attach_vlm_kv")

    def set_prefix_hidden(self, hidden, n_prefix: int, state=None, stream=None):
        """The current prefix from device bf16 hidden states [B][L][P][Hv] (see vla_ae_set_prefix_hidden)."""
        _check(vla_ae_set_prefix_hidden(self.handle, _ptr(hidden), int(n_prefix), _ptr(state), _stream_ptr(stream)),
               "vla_ae_set_prefix_hidden")

    def debug_prefix_kv(self, layer: int, k, v):
        _check(vla_ae_debug_prefix_kv(self.handle, int(layer), _ptr(k), _ptr(v)), "vla_ae_debug_prefix_kv")

    def set_prefix_next(self, k, v, n_prefix: int, state=None, on_device: bool = False, stream=None):
        """Lay out the next cycle's prefix (see vla_ae_set_prefix_next)."""
        _check(vla_ae_set_prefix_next(self.handle, _ptr(k), _ptr(v), int(n_prefix), _ptr(state), int(on_device),
                                      _stream_ptr(stream)), "vla_ae_set_prefix_next")

    def denoise_stale(self, noise, steps: int, n_stale: int, out, stream=None):
        """Steps [0, n_stale) on the current prefix, the rest on the next one (see vla_ae_denoise_stale)."""
        _check(vla_ae_denoise_stale(self.handle, _ptr(noise), int(steps), int(n_stale), _ptr(out),
                                    _stream_ptr(stream)), "vla_ae_denoise_stale")

    def denoise_sched(self, noise, t_grid: Sequence[float], out, stream=None):
        """Euler along the time grid t_grid[0] > ... > t_grid[n] (n steps)."""
        g = (ctypes.c_float * len(t_grid))(*[float(t) for t in t_grid])
        _check(vla_ae_denoise_sched(self.handle, _ptr(noise), g, len(t_grid) - 1, _ptr(out), _stream_ptr(stream)),
               "vla_ae_denoise_sched")

    def denoise_host(self, noise_host, steps: int, out_host, stream=None):
        _check(vla_ae_denoise_host(self.handle, _ptr(noise_host), int(steps), _ptr(out_host), _stream_ptr(stream)),
               "vla_ae_denoise_host")

    def status(self) -> int:
        return vla_ae_status(self.handle)

    def query(self, what: int, arg: int = 0) -> int:
        v = ctypes.c_longlong()
        _check(vla_ae_query(self.handle, what, arg, ctypes.byref(v)), "vla_ae_query")
        return v.value

    def debug_layer(self, layer: int, step: int, steps: int, h_in, h_out, trace: Optional[Dict[str, object]] = None):
        tr = None
        if trace:
            tr = VlaAeTrace(**{k: _ptr(trace.get(k)) for k, _ in VlaAeTrace._fields_})
        _check(vla_ae_debug_layer(self.handle, layer, step, steps, _ptr(h_in), _ptr(h_out),
                                  ctypes.byref(tr) if tr is not None else None), "vla_ae_debug_layer")

    def debug_velocity(self, step: int, steps: int, x, v):
        _check(vla_ae_debug_velocity(self.handle, step, steps, _ptr(x), _ptr(v)), "vla_ae_debug_velocity")

    def debug_weight(self, layer: int, which: int, w_host, scales_host=None):
        _check(vla_ae_debug_weight(self.handle, layer, which, _ptr(w_host), _ptr(scales_host)), "vla_ae_debug_weight")

    def debug_wait_probe(self, attempts: int):
        _check(vla_ae_debug_wait_probe(self.handle, int(attempts)), "vla_ae_debug_wait_probe")

    def set_engine(self, engine: int):
        """ENGINE_PER_OP, ENGINE_PERSISTENT (raises EUNSUPPORTED where it is unavailable) or
        ENGINE_AUTO (the first whole loop of a step count times both and keeps the faster)."""
        _check(vla_ae_set_engine(self.handle, engine), "vla_ae_set_engine")

    @property
    def engine(self) -> int:
        return self.query(Q_ENGINE)

    def bench_op(self, op: int, count: int, steps: int, stream=None):
        _check(vla_ae_bench_op(self.handle, op, count, steps, _stream_ptr(stream)), "vla_ae_bench_op")

    def close(self):
        if getattr(self, "handle", None):
            vla_ae_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
