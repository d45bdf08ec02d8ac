"""GPU parity at the full workload sizes (StarVLA-shaped, pi0.5-shaped, FP8 pi0.5-shaped), in the
launch configuration the benchmark times, against the CPU oracle on the same seeded inputs.

The oracle computes every output here (a full loop is a few seconds of BLAS on the host), so
the comparison covers all actions, plus teacher-forced layers at the first and last Euler step.
"""

import numpy as np
import pytest

import oracle
from synth import config
from tests.gpu_util import Case, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    import __graft_entry__
    __graft_entry__._build_module().build_library()
    yield


def _teacher_forced(c, step, layers):
    import torch
    d = c.d
    traces = c.oracle_layer_traces(step, d.steps)
    out = {}
    for layer in layers:
        h_in = np.concatenate([traces[b][layer]["h_in"] for b in range(d.batch)])
        hin = torch.tensor(h_in, dtype=torch.float32, device="cuda")
        hout = torch.empty_like(hin)
        c.ae.debug_layer(layer, step, d.steps, hin, hout)
        torch.cuda.synchronize()
        ref = np.concatenate([traces[b][layer]["h_out"] for b in range(d.batch)])
        out[layer] = rel_err(hout.cpu().numpy(), ref)
    return out


@pytest.mark.parametrize("name", ["starvla", "pi05"])
def test_full_size_bf16(name):
    import flow_matching_action_euler_b200 as fm
    c = Case(config(name))
    try:
        assert c.ae.engine == fm.ENGINE_PER_OP       # the default, what the benchmark times
        c.ae.set_engine(fm.ENGINE_PERSISTENT)
        got = c.denoise()
        ref = c.oracle_denoise()
        assert rel_err(got, ref) <= 2e-2
        L = c.d.n_layers
        for step in (0, c.d.steps - 1):
            errs = _teacher_forced(c, step, [0, L // 2, L - 1])
            assert max(errs.values()) <= 1e-2, (step, errs)
        # the per-op engine on the same handle
        c.ae.set_engine(fm.ENGINE_PER_OP)
        per_op = c.denoise()
        assert rel_err(per_op, ref) <= 2e-2
        assert rel_err(per_op, got) <= 5e-3
        assert max(_teacher_forced(c, 0, [L - 1]).values()) <= 1e-2
        # velocity at step 0 (x_0 = noise)
        import torch
        x0 = oracle.bf16_to_f64(c.x["noise"])
        v = torch.empty(x0.shape, dtype=torch.float32, device="cuda")
        c.ae.debug_velocity(0, c.d.steps, torch.tensor(x0, dtype=torch.float32, device="cuda"), v)
        noise, st, kp, vp = c.sample_inputs(0)
        vref = oracle.velocity(noise, 1.0, st, c.W, kp, vp, c.d)
        assert rel_err(v.cpu().numpy()[0], vref) <= 2e-2
    finally:
        c.close()


@pytest.mark.parametrize("wtype,steps", [("pi05_fp8", 1), ("pi05_fp8", 10), ("pi05_int8", 1), ("pi05_int8", 10),
                                         ("pi05_int4", 1), ("pi05_int4", 10)])
def test_full_size_fp8(wtype, steps):
    c = Case(config(wtype, steps=steps))
    try:
        got = c.denoise()
        ref_q = c.oracle_denoise()
        assert rel_err(got, ref_q) <= 2e-2
        ref_bf16 = c.oracle_denoise(W=oracle.OracleWeights(c.w, c.d, quantized=False))
        # 8-bit formats within 5e-2 of the bf16-weight oracle; int4 (W4A16) is looser
        assert rel_err(got, ref_bf16) <= (0.25 if c.d.wtype == "int4_g128" else 5e-2)
    finally:
        c.close()


def test_starvla_int4_several_k_tiles():
    """StarVLA-shaped loop (1 Euler step) on INT4 weights.  Its down-projection (1536 rows,
    K = 4096: 16 packed k-tiles) cannot give every K split a single packed tile inside one wave of
    CTAs, so each CTA walks several k-tiles of widened weights: the operand k-blocks of each must
    follow the tile's width (4 k-blocks per int4 tile)."""
    import flow_matching_action_euler_b200 as fm
    c = Case(config("starvla", wtype="int4_g128", steps=1))
    try:
        s_down = (c.ae.query(fm.Q_SPLITS) >> 24) & 0xFF
        assert 16 > s_down                            # more packed k-tiles than splits
        got = c.denoise()
        assert rel_err(got, c.oracle_denoise()) <= 2e-2
    finally:
        c.close()


def test_pi05_one_step_variant():
    """The one-step action generation of the APXInf article on the pi0.5 shape: grid {1, 0}."""
    import torch
    c = Case(config("pi05"))
    try:
        noise = torch.from_numpy(c.x["noise"].view(np.int16)).cuda()
        out = torch.empty((1, c.d.n_action_tokens, c.d.action_dim), dtype=torch.float32, device="cuda")
        c.ae.denoise_sched(noise, [1.0, 0.0], out)
        torch.cuda.synchronize()
        assert c.ae.status() == 0
        ref = c.oracle_denoise(t_grid=[1.0, 0.0])
        assert rel_err(out.cpu().numpy(), ref) <= 2e-2
        assert np.array_equal(out.cpu().numpy(), c.denoise(1))   # the same grid as 1 uniform step
    finally:
        c.close()


@pytest.mark.parametrize("batch", [4, 16, 64])
def test_starvla_batch_sweep_sampled(batch):
    c = Case(config("starvla", batch=batch))
    try:
        got = c.denoise()
        samples = [0, batch - 1]
        ref = c.oracle_denoise(samples=samples)
        assert rel_err(got[samples], ref) <= 2e-2
    finally:
        c.close()
