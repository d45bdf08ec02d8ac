"""The C-ABI library loads, exports every declared symbol, and rejects bad arguments on the host.

No compute call is made here: argument validation happens before any CUDA call, so these
run without a GPU.
"""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vla_ae.h")


@pytest.fixture(scope="module")
def fm():
    import __graft_entry__
    b = __graft_entry__._build_module()
    b.build_library()
    import flow_matching_action_euler_b200 as fm
    return fm


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vla_ae_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("vla_ae_create", "vla_ae_set_prefix", "vla_ae_denoise", "vla_ae_destroy",
                     "vla_ae_status", "vla_ae_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(fm):
    lib = ctypes.CDLL(fm.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_strerror_codes(fm):
    assert fm.vla_ae_strerror(0) == b"ok"
    assert fm.vla_ae_strerror(fm.EINVAL) == b"invalid argument"
    assert fm.vla_ae_strerror(fm.ENOPREFIX) == b"prefix not set"
    assert fm.vla_ae_strerror(12345) == b"unknown error"


def _dims(fm, **kw):
    base = dict(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, inter=704, t_emb_dim=256,
                action_dim=7, n_action_tokens=16, has_state_token=0, max_prefix=64, batch=1)
    base.update(kw)
    d = fm.VlaAeDims()
    for k, v in base.items():
        setattr(d, k, v)
    d.rope_theta = 10000.0
    d.rms_eps = 1e-6
    d.wtype = kw.get("wtype", 0)
    return d


@pytest.mark.parametrize("bad", [
    dict(n_layers=0), dict(hidden=250), dict(inter=700 + 3), dict(n_q_heads=3, n_kv_heads=2),
    dict(action_dim=65), dict(has_state_token=2), dict(batch=0), dict(max_prefix=-1),
    dict(batch=300, n_action_tokens=16), dict(wtype=7), dict(t_emb_dim=255),
])
def test_create_rejects_bad_dims_before_touching_cuda(fm, bad):
    d = _dims(fm, **bad)
    w = fm.VlaAeWeights()
    h = ctypes.c_void_p()
    assert fm.vla_ae_create(ctypes.byref(d), ctypes.byref(w), ctypes.byref(h)) == fm.EINVAL
    assert not h.value


def test_unsupported_head_dim(fm):
    d = _dims(fm, head_dim=96)
    w = fm.VlaAeWeights()
    h = ctypes.c_void_p()
    assert fm.vla_ae_create(ctypes.byref(d), ctypes.byref(w), ctypes.byref(h)) == fm.EUNSUPPORTED


def test_null_arguments(fm):
    h = ctypes.c_void_p()
    assert fm.vla_ae_create(None, None, ctypes.byref(h)) == fm.EINVAL
    assert fm.vla_ae_create(ctypes.byref(_dims(fm)), None, ctypes.byref(h)) == fm.EINVAL
    assert fm.vla_ae_denoise(None, None, 4, None, None) == fm.EINVAL
    assert fm.vla_ae_denoise_host(None, None, 4, None, None) == fm.EINVAL
    assert fm.vla_ae_set_prefix(None, None, None, 0, None, 0, None) == fm.EINVAL
    v = ctypes.c_longlong()
    assert fm.vla_ae_query(None, 1, 4, ctypes.byref(v)) == fm.EINVAL
    assert fm.vla_ae_status(None) == fm.EINVAL
    assert fm.vla_ae_debug_layer(None, 0, 0, 1, None, None, None) == fm.EINVAL
    assert fm.vla_ae_debug_velocity(None, 0, 1, None, None) == fm.EINVAL
    assert fm.vla_ae_debug_weight(None, 0, 0, None, None) == fm.EINVAL
    assert fm.vla_ae_debug_wait_probe(None, 10) == fm.EINVAL
    assert fm.vla_ae_set_prefix_static(None, None, None, 0, None, None) == fm.EINVAL
    g = (ctypes.c_float * 3)(1.0, 0.5, 0.0)
    assert fm.vla_ae_denoise_sched(None, None, g, 2, None, None) == fm.EINVAL
    assert fm.vla_ae_set_engine(None, fm.ENGINE_PER_OP) == fm.EINVAL
    assert fm.vla_ae_set_prefix_next(None, None, None, 0, None, 0, None) == fm.EINVAL
    assert fm.vla_ae_denoise_stale(None, None, 4, 2, None, None) == fm.EINVAL
    assert fm.vla_ae_attach_vlm_kv(None, None) == fm.EINVAL
    assert fm.vla_ae_set_prefix_hidden(None, None, 1, None, None) == fm.EINVAL
    assert fm.vla_ae_debug_prefix_kv(None, 0, None, None) == fm.EINVAL
    fm.vla_ae_destroy(None)   # no-op


def test_binding_is_marshalling_only():
    """The binding module holds no arithmetic of the method and never imports the oracle."""
    src = open(os.path.join(ROOT, "flow_matching_action_euler_b200", "__init__.py")).read()
    for banned in ("import oracle", "from oracle", "import numpy", "import torch", "import synth"):
        assert banned not in src, banned
