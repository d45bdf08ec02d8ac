"""Helpers shared by the GPU parity tests: build a handle from the synthetic inputs, run the
oracle on the same inputs, and measure the relative error the tolerances are stated in."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from synth import abi_dims, generate_inputs, generate_weights


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| over the whole tensor (batch included)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def bits_to_cuda(a: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> a CUDA int16 tensor holding the same bits."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


class Case:
    """One workload on the GPU plus its oracle."""

    def __init__(self, d, seed: int = 0, n_prefix: int | None = None, max_prefix: int | None = None):
        import flow_matching_action_euler_b200 as fm
        self.d = d
        self.P = d.n_prefix if n_prefix is None else n_prefix
        self.w = generate_weights(d, seed)
        self.x = generate_inputs(d, seed, n_prefix=self.P)
        self.ae = fm.ActionExpert(abi_dims(d, max_prefix=max_prefix if max_prefix is not None else d.n_prefix),
                                  self.w)
        self.ae.set_prefix(self.x["k"] if self.P else None, self.x["v"] if self.P else None, self.P,
                           self.x.get("state"))
        self.W = oracle.OracleWeights(self.w, d, quantized=d.wtype)

    def denoise(self, steps: int | None = None) -> np.ndarray:
        d = self.d
        steps = d.steps if steps is None else steps
        noise = bits_to_cuda(self.x["noise"])
        out = torch.empty((d.batch, d.n_action_tokens, d.action_dim), dtype=torch.float32, device="cuda")
        self.ae.denoise(noise, steps, out)
        torch.cuda.synchronize()
        assert self.ae.status() == 0
        return out.cpu().numpy()

    def oracle_denoise(self, steps: int | None = None, samples=None, W=None, t_grid=None) -> np.ndarray:
        return oracle.denoise_batch(self.w, self.x, self.d, n_steps=steps, samples=samples,
                                    W=self.W if W is None else W, t_grid=t_grid)

    def sample_inputs(self, b: int):
        x = self.x
        st = oracle.bf16_to_f64(x["state"][b]) if self.d.has_state_token else None
        return (oracle.bf16_to_f64(x["noise"][b]), st, oracle.bf16_to_f64(x["k"][b]), oracle.bf16_to_f64(x["v"][b]))

    def oracle_state_at(self, b: int, step: int, steps: int) -> np.ndarray:
        """x_step of sample b along the oracle's own trajectory."""
        noise, st, kp, vp = self.sample_inputs(b)
        ts, dt = oracle.t_schedule(steps)
        xk = noise
        for k in range(step):
            xk = xk + dt * oracle.velocity(xk, ts[k], st, self.W, kp, vp, self.d)
        return xk

    def oracle_layer_traces(self, step: int, steps: int):
        """Per sample: list over layers of the oracle's intermediates at x_step."""
        ts, _ = oracle.t_schedule(steps)
        traces = []
        for b in range(self.d.batch):
            noise, st, kp, vp = self.sample_inputs(b)
            xk = self.oracle_state_at(b, step, steps)
            tr = []
            oracle.velocity(xk, ts[step], st, self.W, kp, vp, self.d, layer_trace=tr)
            traces.append(tr)
        return traces

    def close(self):
        self.ae.close()
