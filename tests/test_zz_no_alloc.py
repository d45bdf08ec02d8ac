"""The allocation-free prefix upload (vla_ae_set_prefix_static) against the allocating one.

vla_ae_set_prefix_static is for callers that cannot allocate device memory while they run (a
control loop that must not pay allocator latency every cycle, or code running during CUDA-graph
capture).  It stages the prefix through a fixed device array compiled into the library instead
of buffers it allocates.  Called through the C ABI twice in a row (two different prefixes), the
denoise results after it must match those after vla_ae_set_prefix with the same host inputs.
This file is collected last so that a run stopping at the first failure has run everything else.
"""

import numpy as np
import pytest
import torch

import oracle
from synth import abi_dims, config, generate_inputs, generate_weights

pytestmark = pytest.mark.gpu

FINAL_TOL = 2e-2


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.fixture(scope="module")
def fm(cuda_device):
    import __graft_entry__
    __graft_entry__._build_module().build_library()
    import flow_matching_action_euler_b200 as fm
    return fm


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("tiny", 3), ("starvla", 2)])
def test_set_prefix_static_matches_allocating_path(fm, name, batch):
    d = config(name, batch=batch)
    w = generate_weights(d, 0)
    first = generate_inputs(d, seed=0)
    second = generate_inputs(d, seed=7)
    ae = fm.ActionExpert(abi_dims(d), w)
    try:
        out = torch.empty((d.batch, d.n_action_tokens, d.action_dim), dtype=torch.float32, device="cuda")

        def run(inputs, static):
            state = inputs.get("state")
            if static:
                ae.set_prefix_static(inputs["k"], inputs["v"], d.n_prefix, state)
            else:
                ae.set_prefix(inputs["k"], inputs["v"], d.n_prefix, state)
            ae.denoise(torch.from_numpy(inputs["noise"].view(np.int16)).cuda(), d.steps, out)
            torch.cuda.synchronize()
            assert ae.status() == 0
            return out.cpu().numpy().copy()

        for inputs in (first, second):            # two calls in a row, different prefixes
            ref = run(inputs, static=False)
            got = run(inputs, static=True)
            assert _rel(got, ref) <= 1e-6
            assert np.array_equal(got, ref)       # same kernels, same inputs: bit-identical
        # and the static path on its own still matches the oracle on the last prefix
        sample = [0] if batch == 1 else [0, batch - 1]
        want = oracle.denoise_batch(w, second, d, samples=sample)
        assert _rel(got[sample], want) <= FINAL_TOL
    finally:
        ae.close()


def test_set_prefix_static_rejects_oversized_prefix(fm):
    # one layer of K+V for the batch must fit the 16 MiB staging array: 32 x 300 x 4 x 128 x 4 B > 16 MiB
    d = config("starvla", batch=32, n_layers=1)
    w = generate_weights(d, 0)
    ae = fm.ActionExpert(abi_dims(d), w)
    try:
        k = np.zeros((32, 1, 300, 4, 128), np.uint16)
        state = np.zeros((32, d.action_dim), np.uint16)
        with pytest.raises(fm.VlaAeError) as err:
            ae.set_prefix_static(k, k, 300, state)
        assert err.value.code == fm.EINVAL
    finally:
        ae.close()
