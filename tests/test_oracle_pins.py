"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test ties an oracle function to something other than itself: a closed form, an
invariant, a library routine computing the same textbook operation, brute force on tiny
inputs, or a golden table written from a format definition.
"""

import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch
import torch.nn.functional as F

import oracle
from oracle import fp8 as ofp8
from synth import config, generate_weights, generate_inputs, f32_to_bf16_bits, bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------- Euler sampler

def _linear_field(n=7, seed=0):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((n, n))
    a = a / np.linalg.norm(a, 2)            # spectral norm 1
    b = rng.standard_normal(n)
    x0 = rng.standard_normal(n)
    return a, b, x0


@pytest.mark.parametrize("n_steps", [1, 2, 4, 10, 37])
def test_euler_linear_field_closed_form(n_steps):
    a, b, x0 = _linear_field()
    got = oracle.euler_integrate(x0, n_steps, lambda x, t: a @ x + b)
    dt = -1.0 / n_steps
    m = np.eye(7) + dt * a
    want = np.linalg.matrix_power(m, n_steps) @ x0
    for j in range(n_steps):
        want = want + np.linalg.matrix_power(m, j) @ (dt * b)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_euler_converges_to_exact_flow_first_order():
    a, b, x0 = _linear_field(seed=3)
    ea = scipy.linalg.expm(-a)
    exact = ea @ x0 + np.linalg.solve(a, (ea - np.eye(7)) @ b)
    errs = []
    for n in (64, 128, 256, 512):
        got = oracle.euler_integrate(x0, n, lambda x, t: a @ x + b)
        errs.append(np.max(np.abs(got - exact)))
    ratios = [errs[i] / errs[i + 1] for i in range(3)]
    for r in ratios:
        assert 1.8 < r < 2.2, (errs, ratios)           # global error O(|dt|)
    # the Euler bound |err| <= |dt| * C with C of order ||A|| e^{||A||} (||b|| + ||x||)
    assert errs[0] < 64 ** -1 * 50


def test_euler_zero_field_and_single_step():
    _, b, x0 = _linear_field(seed=5)
    got = oracle.euler_integrate(x0, 8, lambda x, t: b)
    np.testing.assert_allclose(got, x0 - b, rtol=0, atol=1e-14)
    seen = []

    def v(x, t):
        seen.append(t)
        return np.sin(x) + t

    got1 = oracle.euler_integrate(x0, 1, v)
    assert seen == [1.0]
    assert np.array_equal(got1, x0 - (np.sin(x0) + 1.0))


def test_euler_time_grid_golden():
    with open(os.path.join(GOLDEN, "euler_schedule.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for r in rows:
        n, dt, ts = int(r[0]), float(r[1]), [float(x) for x in r[2:]]
        got_ts, got_dt = oracle.t_schedule(n)
        assert got_dt == dt
        np.testing.assert_allclose(got_ts, ts, rtol=0, atol=1e-15)
        seen = []
        oracle.euler_integrate(np.zeros(1), n, lambda x, t: seen.append(t) or np.zeros(1))
        np.testing.assert_allclose(seen, ts, rtol=0, atol=1e-15)


# ----------------------------------------------------------------- Euler along a time grid

def test_euler_grid_uniform_matches_fixed_step():
    a, b, x0 = _linear_field(seed=7)
    for n in (1, 3, 10):
        got = oracle.euler_integrate_grid(x0, oracle.uniform_grid(n), lambda x, t: a @ x + b + t)
        want = oracle.euler_integrate(x0, n, lambda x, t: a @ x + b + t)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_euler_grid_skipping_equals_velocity_cache():
    """Dropping grid points = reusing the last computed velocity over the dropped steps."""
    a, b, x0 = _linear_field(seed=8)
    field = lambda x, t: np.tanh(a @ x) + b * t
    n = 10
    keep = {0, 1, 2, 6, 9}                      # velocities recomputed only at these steps
    x, v = np.array(x0), None
    for k in range(n):                           # brute force: the uniform loop with a cache
        if k in keep:
            v = field(x, 1.0 - k / n)
        x = x + (-1.0 / n) * v
    grid = [1.0 - k / n for k in sorted(keep)] + [0.0]
    got = oracle.euler_integrate_grid(x0, grid, field)
    np.testing.assert_allclose(got, x, rtol=1e-13, atol=1e-13)


def test_euler_grid_converges_first_order_on_a_graded_grid():
    a, b, x0 = _linear_field(seed=3)
    ea = scipy.linalg.expm(-a)
    exact = ea @ x0 + np.linalg.solve(a, (ea - np.eye(7)) @ b)
    errs = []
    for n in (64, 128, 256):
        grid = [(1.0 - k / n) ** 2 for k in range(n + 1)]      # steps from 2/n down to 1/n^2
        errs.append(np.max(np.abs(oracle.euler_integrate_grid(x0, grid, lambda x, t: a @ x + b) - exact)))
    for r in (errs[0] / errs[1], errs[1] / errs[2]):
        assert 1.8 < r < 2.2, errs


def test_euler_grid_one_step_and_order_of_times():
    _, b, x0 = _linear_field(seed=9)
    seen = []

    def v(x, t):
        seen.append(t)
        return np.cos(x) * t

    got = oracle.euler_integrate_grid(x0, [1.0, 0.0], v)
    assert seen == [1.0]
    assert np.array_equal(got, x0 - np.cos(x0))
    seen.clear()
    oracle.euler_integrate_grid(x0, [0.9, 0.7, 0.2, -0.1], v)
    assert seen == [0.9, 0.7, 0.2]
    got = oracle.euler_integrate_grid(x0, [1.0, 0.6, 0.25, 0.0], lambda x, t: b)
    np.testing.assert_allclose(got, x0 - b, rtol=0, atol=1e-14)


@pytest.mark.parametrize("grid", [[1.0], [1.0, 1.0], [0.2, 0.5], [1.0, float("nan"), 0.0], [1.0, 0.5, 0.5, 0.0]])
def test_euler_grid_rejects_bad_grids(grid):
    with pytest.raises(ValueError):
        oracle.check_t_grid(grid)


# ----------------------------------------------------------------- Euler with a switched field

@pytest.mark.parametrize("n_steps,n_stale", [(4, 2), (10, 5), (7, 1), (7, 6)])
def test_euler_switch_linear_fields_closed_form(n_steps, n_stale):
    a1, b1, x0 = _linear_field(seed=11)
    a2, b2, _ = _linear_field(seed=12)
    got = oracle.euler_integrate_switch(x0, n_steps, n_stale, lambda x, t: a1 @ x + b1, lambda x, t: a2 @ x + b2)
    dt = -1.0 / n_steps
    m1, m2 = np.eye(7) + dt * a1, np.eye(7) + dt * a2
    mp = np.linalg.matrix_power
    xs = mp(m1, n_stale) @ x0 + sum((mp(m1, j) @ (dt * b1) for j in range(n_stale)), np.zeros(7))
    want = mp(m2, n_steps - n_stale) @ xs + sum((mp(m2, j) @ (dt * b2) for j in range(n_steps - n_stale)), np.zeros(7))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_euler_switch_extremes_reduce_to_one_field():
    a1, b1, x0 = _linear_field(seed=13)
    f1 = lambda x, t: np.tanh(a1 @ x) + t
    f2 = lambda x, t: np.sin(x) - b1
    for n in (1, 4):
        assert np.array_equal(oracle.euler_integrate_switch(x0, n, n, f1, f2), oracle.euler_integrate(x0, n, f1))
        assert np.array_equal(oracle.euler_integrate_switch(x0, n, 0, f1, f2), oracle.euler_integrate(x0, n, f2))
    with pytest.raises(ValueError):
        oracle.euler_integrate_switch(x0, 4, 5, f1, f2)


# ----------------------------------------------------------------- time embedding

def test_timestep_embedding_t0_and_identity():
    e = oracle.timestep_embedding(0.0, 256)
    assert np.array_equal(e, np.concatenate([np.ones(128), np.zeros(128)]))
    for t in (1.0, 0.75, 0.1, 0.333):
        e = oracle.timestep_embedding(t, 256)
        # cos^2 + sin^2 = 1 pairs element i of each half at the same frequency
        np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-14)
        # first frequency is 1: a_0 = 1000 t
        assert math.isclose(e[0], math.cos(1000.0 * t), abs_tol=1e-12)
        assert math.isclose(e[128], math.sin(1000.0 * t), abs_tol=1e-12)
    # frequencies form a geometric series from 1 down to 10000^(-127/128)
    t = 1e-4
    e = oracle.timestep_embedding(t, 256)
    ang = np.arctan2(e[128:], e[:128]) / (1000.0 * t)
    ratio = ang[1:] / ang[:-1]
    np.testing.assert_allclose(ratio, 10000.0 ** (-1.0 / 128), rtol=1e-9)


def test_silu_values():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    z = RNG.standard_normal(100) * 4
    np.testing.assert_allclose(oracle.silu(z), F.silu(torch.tensor(z)).numpy(), rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------- RMSNorm / modulate

def test_rms_norm_unit_rms_and_scale_invariance():
    h = RNG.standard_normal((5, 96)) * 3.0
    y = oracle.rms_norm(h, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-12)
    np.testing.assert_allclose(oracle.rms_norm(7.5 * h, eps=0.0), y, rtol=1e-12, atol=1e-13)
    # textbook routine: torch's rms_norm with the same eps and no affine weight
    want = F.rms_norm(torch.tensor(h), (96,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rms_norm(h, 1e-6), want, rtol=1e-12, atol=1e-13)


def test_modulate_identity_and_form():
    u = RNG.standard_normal((3, 8))
    z = np.zeros(8)
    assert np.array_equal(oracle.modulate(u, z, z), u)
    np.testing.assert_allclose(oracle.modulate(u, z, -np.ones(8)), 0.0)      # (1 + scale) form
    s = RNG.standard_normal(8)
    np.testing.assert_allclose(oracle.modulate(u, s, z), u + s)


# ----------------------------------------------------------------- RoPE

@pytest.mark.parametrize("hd", [8, 64, 256])
def test_rope_invariants(hd):
    x = RNG.standard_normal((6, 3, hd))
    pos = np.arange(6) + 11.0
    y = oracle.rope_half(x, pos)
    half = hd // 2
    np.testing.assert_allclose(x[..., :half] ** 2 + x[..., half:] ** 2,
                               y[..., :half] ** 2 + y[..., half:] ** 2, rtol=1e-12)
    np.testing.assert_allclose(oracle.rope_half(x, np.zeros(6)), x, rtol=0, atol=0)
    # complex form: z_i = x_i + i x_{i+hd/2} rotated by e^{i theta}, theta = p * 10000^(-2i/hd)
    z = x[..., :half] + 1j * x[..., half:]
    th = pos[:, None, None] * 10000.0 ** (-2.0 * np.arange(half) / hd)[None, None, :]
    zr = z * np.exp(1j * th)
    np.testing.assert_allclose(y[..., :half], zr.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y[..., half:], zr.imag, rtol=1e-12, atol=1e-12)


def test_rope_relative_position():
    hd = 32
    q = RNG.standard_normal((1, 1, hd))
    k = RNG.standard_normal((1, 1, hd))
    for m, n, s in ((3, 7, 5), (0, 10, 100), (40, 2, 17)):
        a = np.sum(oracle.rope_half(q, np.array([m * 1.0])) * oracle.rope_half(k, np.array([n * 1.0])))
        b = np.sum(oracle.rope_half(q, np.array([m + s * 1.0])) * oracle.rope_half(k, np.array([n + s * 1.0])))
        assert math.isclose(a, b, rel_tol=1e-10, abs_tol=1e-12)


# ----------------------------------------------------------------- attention

def _brute_attention(q, k, v):
    """Score matrix written out element by element, kv heads materialised by repetition."""
    T, nq, hd = q.shape
    nkv = k.shape[1]
    k_rep = np.repeat(k, nq // nkv, axis=1)
    v_rep = np.repeat(v, nq // nkv, axis=1)
    out = np.zeros_like(q)
    for h in range(nq):
        for i in range(T):
            s = [sum(q[i, h, d] * k_rep[j, h, d] for d in range(hd)) / math.sqrt(hd)
                 for j in range(k.shape[0])]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            for d in range(hd):
                out[i, h, d] = sum(e[j] * v_rep[j, h, d] for j in range(k.shape[0])) / z
    return out


@pytest.mark.parametrize("nq,nkv", [(4, 2), (4, 1), (4, 4)])
def test_attention_brute_force_and_sdpa(nq, nkv):
    Ts, P, hd = 3, 5, 8
    q = RNG.standard_normal((Ts, nq, hd))
    k = RNG.standard_normal((P + Ts, nkv, hd))
    v = RNG.standard_normal((P + Ts, nkv, hd))
    got = oracle.gqa_attention(q, k, v)
    np.testing.assert_allclose(got, _brute_attention(q, k, v), rtol=1e-12, atol=1e-13)
    want = F.scaled_dot_product_attention(
        torch.tensor(q).permute(1, 0, 2)[None], torch.tensor(k).permute(1, 0, 2)[None],
        torch.tensor(v).permute(1, 0, 2)[None], enable_gqa=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    q = RNG.standard_normal((4, 2, 16))
    k = RNG.standard_normal((9, 1, 16))
    v = np.tile(RNG.standard_normal((1, 1, 16)), (9, 1, 1))     # every V row equal
    np.testing.assert_allclose(oracle.gqa_attention(q, k, v), np.broadcast_to(v[0, 0], (4, 2, 16)),
                               rtol=1e-13, atol=1e-14)
    one = oracle.gqa_attention(q[:1], k[:1], RNG.standard_normal((1, 1, 16)))
    assert one.shape == (1, 2, 16)
    # a single key gets all the weight
    vv = RNG.standard_normal((1, 1, 16))
    np.testing.assert_allclose(oracle.gqa_attention(q, k[:1], vv), np.broadcast_to(vv[0, 0], (4, 2, 16)))


# ----------------------------------------------------------------- linear / SwiGLU

def test_linear_and_swiglu_vs_torch():
    x = RNG.standard_normal((5, 24))
    w = RNG.standard_normal((10, 24))
    b = RNG.standard_normal(10)
    np.testing.assert_allclose(oracle.linear(x, w, b),
                               F.linear(torch.tensor(x), torch.tensor(w), torch.tensor(b)).numpy(),
                               rtol=1e-12, atol=1e-12)
    wg = RNG.standard_normal((7, 24))
    wu = RNG.standard_normal((7, 24))
    tx = torch.tensor(x)
    want = (F.silu(F.linear(tx, torch.tensor(wg))) * F.linear(tx, torch.tensor(wu))).numpy()
    np.testing.assert_allclose(oracle.swiglu(x, wg, wu), want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- FP8 e4m3

def test_e4m3_golden_table():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    for code, val in rows:
        got = ofp8.e4m3_decode(np.array([code], np.uint8))[0]
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), (hex(code), got, val)
            assert ofp8.e4m3_encode(np.array([val]))[0] == code


def test_e4m3_exhaustive_roundtrip_ties_saturation():
    codes = np.arange(256, dtype=np.uint8)
    vals = ofp8.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254
    assert np.array_equal(ofp8.e4m3_encode(vals[finite]), codes[finite])
    # ties: the midpoint between neighbouring positive codes goes to the even mantissa
    pos = np.arange(0, 0x7E)
    lo, hi = ofp8.e4m3_decode(pos.astype(np.uint8)), ofp8.e4m3_decode((pos + 1).astype(np.uint8))
    mid = (lo + hi) / 2
    got = ofp8.e4m3_encode(mid).astype(int)
    want = np.where(pos % 2 == 0, pos, pos + 1)
    assert np.array_equal(got, want)
    # just above / below a midpoint go to the nearer code
    assert np.array_equal(ofp8.e4m3_encode(np.nextafter(mid, np.inf)).astype(int), pos + 1)
    assert np.array_equal(ofp8.e4m3_encode(np.nextafter(mid, -np.inf)).astype(int), pos)
    # saturation
    big = np.array([448.0, 449.0, 464.0, 500.0, 1e6, np.inf, -1e9, -np.inf])
    assert list(ofp8.e4m3_encode(big)) == [0x7E] * 6 + [0xFE] * 2
    assert ofp8.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_e4m3_matches_torch_cast_in_range():
    x = np.concatenate([RNG.standard_normal(20000) * s for s in (0.003, 0.1, 3, 60, 150)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    pos = np.arange(0, 0x7E)
    mids = ((ofp8.e4m3_decode(pos.astype(np.uint8)) + ofp8.e4m3_decode((pos + 1).astype(np.uint8))) / 2)
    x = np.concatenate([x, mids.astype(np.float32), -mids.astype(np.float32)])
    want = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ofp8.e4m3_encode(x), want)


def test_rowwise_quantiser():
    w = (RNG.standard_normal((6, 40)) * 0.02).astype(np.float32)
    w[3] = 0.0
    codes, scales = ofp8.quantize_rowwise_e4m3(w)
    assert scales.dtype == np.float32 and scales[3] == 1.0
    assert np.all(codes[3] == 0)
    for o in (0, 1, 2, 4, 5):
        i = np.argmax(np.abs(w[o]))
        assert codes[o, i] in (0x7E, 0xFE)
    deq = ofp8.dequantize_rowwise_e4m3(codes, scales)
    # e4m3 keeps 3 mantissa bits: relative error of a normal value <= 2^-4
    big = np.abs(w) > scales[:, None] * 2 ** -6
    assert np.all(np.abs(deq - w)[big] <= np.abs(w)[big] * 2 ** -4 + 1e-12)


# ----------------------------------------------------------------- layer / model composition

MICRO = config("tiny", n_layers=2, hidden=64, n_q_heads=4, n_kv_heads=2, head_dim=16, inter=96,
               n_prefix=7, action_dim=5, n_action_tokens=6, has_state_token=1, steps=3)


def _layer_inputs(d, seed=0):
    w = generate_weights(d, seed)
    W = oracle.OracleWeights(w, d)
    x = generate_inputs(d, seed)
    lw = W.layer(0)
    mod = oracle.adaln_table(lw["w_ada"], lw["b_ada"], 0.75, d.t_emb_dim)
    kp = oracle.bf16_to_f64(x["k"][0, 0])
    vp = oracle.bf16_to_f64(x["v"][0, 0])
    h = RNG.standard_normal((d.ts, d.hidden)) * 0.1
    pos = d.n_prefix + np.arange(d.ts, dtype=np.float64)
    return W, lw, mod, kp, vp, h, pos


def test_adaln_table_at_t0_closed_form():
    """At t = 0 the embedding is [cos 0 .. | sin 0 ..] = [1 .. 1 | 0 .. 0], so the modulation is
    SiLU(1) times the row sums of W_ada's first half of columns, plus b_ada (SiLU(1) = 1 / (1 +
    1/e)).  Pins the [cos | sin] order, the SiLU before the projection, W_ada's orientation and
    the bias."""
    rng = np.random.default_rng(21)
    dt_dim, rows = 16, 12
    w = rng.standard_normal((rows, dt_dim))
    b = rng.standard_normal(rows)
    silu1 = 1.0 / (1.0 + math.exp(-1.0))
    want = silu1 * w[:, :dt_dim // 2].sum(axis=1) + b
    np.testing.assert_allclose(oracle.adaln_table(w, b, 0.0, dt_dim), want, rtol=1e-14, atol=1e-14)


def test_layer_zero_gates_is_identity():
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d)
    H = d.hidden
    mod = mod.copy()
    mod[2 * H:3 * H] = 0.0
    mod[5 * H:6 * H] = 0.0
    assert np.array_equal(oracle.dit_layer(h, lw, mod, kp, vp, pos, d), h)


def test_layer_prefix_permutation_invariance():
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d, seed=1)
    perm = np.random.default_rng(9).permutation(kp.shape[0])
    a = oracle.dit_layer(h, lw, mod, kp, vp, pos, d)
    b = oracle.dit_layer(h, lw, mod, kp[perm], vp[perm], pos, d)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    # swapping only K rows (not V) must change the result: the pairing of K and V matters
    c = oracle.dit_layer(h, lw, mod, kp[perm], vp, pos, d)
    assert np.max(np.abs(a - c)) > 1e-6


def test_layer_trace_is_consistent():
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d, seed=2)
    tr = {}
    out = oracle.dit_layer(h, lw, mod, kp, vp, pos, d, tr)
    assert np.array_equal(out, tr["h_out"])
    np.testing.assert_allclose(np.sqrt(np.mean(oracle.rms_norm(h, 0.0) ** 2, axis=1)), 1.0)
    assert tr["q"].shape == (d.ts, d.n_q_heads, d.head_dim)
    assert tr["m"].shape == (d.ts, d.inter)


def test_batch_independence_bitwise_and_determinism():
    d = MICRO.replace(batch=3)
    w = generate_weights(d, 0)
    x = generate_inputs(d, 0)
    full = oracle.denoise_batch(w, x, d)
    d1 = d.replace(batch=1)
    for b in range(3):
        xb = {k: v[b:b + 1] for k, v in x.items()}
        one = oracle.denoise_batch(w, xb, d1)
        assert np.array_equal(one[0], full[b])
    again = oracle.denoise_batch(w, x, d)
    assert np.array_equal(again, full)


def test_velocity_with_closed_gates_closed_form():
    """All adaLN gates and the final modulation zero: every DiT layer is the identity, so the
    velocity of action row j is W_out RMSNorm(W_in x_j + b_in) + b_out, the state row (first) being
    dropped.  Written here with einsum on that closed form; pins the in/out projection
    orientation, the per-row final norm, the biases and which row is dropped."""
    d = MICRO
    w = generate_weights(d, 0)
    x = generate_inputs(d, 0)
    H = d.hidden
    w = dict(w)
    w["layers"] = [dict(lw) for lw in w["layers"]]
    for lw in w["layers"]:
        for key in ("w_ada", "b_ada"):
            a = lw[key].copy()
            a[2 * H:3 * H] = 0                                   # gate_a (bf16 +0)
            a[5 * H:6 * H] = 0                                   # gate_m
            lw[key] = a
    w["w_fada"] = np.zeros_like(w["w_fada"])
    w["b_fada"] = np.zeros_like(w["b_fada"])
    W = oracle.OracleWeights(w, d)
    xs = oracle.bf16_to_f64(x["noise"][0])
    st = oracle.bf16_to_f64(x["state"][0])
    kp, vp = oracle.bf16_to_f64(x["k"][0]), oracle.bf16_to_f64(x["v"][0])
    got = oracle.velocity(xs, 0.4, st, W, kp, vp, d)
    top = {k: oracle.bf16_to_f64(w[k]) for k in ("w_in", "b_in", "w_out", "b_out")}
    h = np.einsum("ha,ta->th", top["w_in"], xs) + top["b_in"]
    u = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + d.rms_eps)
    want = np.einsum("ah,th->ta", top["w_out"], u) + top["b_out"]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    # the prefix and the time no longer matter
    np.testing.assert_allclose(oracle.velocity(xs, 0.9, st, W, kp + 1.0, vp * 2.0, d), got, rtol=1e-12, atol=1e-13)


def test_single_step_is_one_euler_update():
    d = MICRO
    w = generate_weights(d, 0)
    x = generate_inputs(d, 0)
    W = oracle.OracleWeights(w, d)
    noise = oracle.bf16_to_f64(x["noise"][0])
    state = oracle.bf16_to_f64(x["state"][0])
    kp, vp = oracle.bf16_to_f64(x["k"][0]), oracle.bf16_to_f64(x["v"][0])
    v = oracle.velocity(noise, 1.0, state, W, kp, vp, d)
    got = oracle.denoise(noise, state, W, kp, vp, d, 1)
    assert np.array_equal(got, noise - v)


# ----------------------------------------------------------------- input preparation

def test_synth_bf16_rounding_matches_torch():
    z = np.concatenate([RNG.standard_normal(50000).astype(np.float32) * s for s in (1e-3, 0.02, 1, 300)])
    want = torch.tensor(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f32_to_bf16_bits(z), want)
    back = bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.tensor(z).to(torch.bfloat16).float().numpy())


def test_layer_self_token_permutation_equivariance():
    """No mask: permuting the self tokens together with their positions permutes the output."""
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d, seed=3)
    perm = np.array([4, 0, 6, 2, 1, 5, 3])[:d.ts]
    a = oracle.dit_layer(h, lw, mod, kp, vp, pos, d)
    b = oracle.dit_layer(h[perm], lw, mod, kp, vp, pos[perm], d)
    np.testing.assert_allclose(b, a[perm], rtol=1e-12, atol=1e-13)


def test_layer_branch_isolation_under_zero_gates():
    """gate_a = 0 cuts the attention branch; gate_m = 0 cuts the MLP branch (adaLN-Zero)."""
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d, seed=4)
    H = d.hidden
    rng = np.random.default_rng(11)

    def perturbed(lw_, keys):
        out = dict(lw_)
        for k_ in keys:
            out[k_] = lw_[k_] + rng.standard_normal(lw_[k_].shape) * 0.05
        return out

    m_a = mod.copy()
    m_a[2 * H:3 * H] = 0.0                   # no attention branch
    base = oracle.dit_layer(h, lw, m_a, kp, vp, pos, d)
    alt = oracle.dit_layer(h, perturbed(lw, ("wq", "wk", "wv", "wo")), m_a,
                           kp + 1.0, vp - 1.0, pos, d)
    np.testing.assert_allclose(alt, base, rtol=1e-13, atol=1e-14)
    m_a2 = m_a.copy()
    m_a2[0:2 * H] += 0.3                     # attention shift/scale only feed that branch
    np.testing.assert_allclose(oracle.dit_layer(h, lw, m_a2, kp, vp, pos, d), base, rtol=1e-13, atol=1e-14)

    m_m = mod.copy()
    m_m[5 * H:6 * H] = 0.0                   # no MLP branch
    base = oracle.dit_layer(h, lw, m_m, kp, vp, pos, d)
    alt = oracle.dit_layer(h, perturbed(lw, ("wg", "wu", "wd")), m_m, kp, vp, pos, d)
    np.testing.assert_allclose(alt, base, rtol=1e-13, atol=1e-14)
    m_m2 = m_m.copy()
    m_m2[3 * H:5 * H] += 0.3
    np.testing.assert_allclose(oracle.dit_layer(h, lw, m_m2, kp, vp, pos, d), base, rtol=1e-13, atol=1e-14)
    # and each branch does contribute when its gate is on
    assert np.max(np.abs(oracle.dit_layer(h, lw, mod, kp, vp, pos, d) - base)) > 1e-6


def test_layer_uniform_attention_closed_form():
    """W_q = 0 makes every score 0, so each query head's softmax is uniform over the P + Ts keys
    and its output is the plain mean of its kv group's value rows: the prefix V rows and the
    self rows v = W_v u (not rotated), u = RMSNorm(h) (1 + scale_a) + shift_a.  With the MLP gate
    closed the layer is then h + gate_a * W_o o, written out here with einsum on that closed
    form (no softmax), which pins the adaLN chunk order of the attention branch, the GQA
    head-to-group map and the prefix + self key set."""
    d = MICRO
    W, lw, mod, kp, vp, h, pos = _layer_inputs(d, seed=5)
    H, hd, nq, nkv = d.hidden, d.head_dim, d.n_q_heads, d.n_kv_heads
    lw = dict(lw)
    lw["wq"] = np.zeros_like(lw["wq"])
    mod = mod.copy()
    mod[5 * H:6 * H] = 0.0                                    # gate_m: MLP branch off
    shift_a, scale_a, gate_a = mod[0:H], mod[H:2 * H], mod[2 * H:3 * H]
    ms = np.mean(h * h, axis=1, keepdims=True)
    u = h / np.sqrt(ms + d.rms_eps) * (1.0 + scale_a) + shift_a
    v_self = np.einsum("ok,tk->to", lw["wv"], u).reshape(d.ts, nkv, hd)
    v_all = np.concatenate([vp, v_self], axis=0)              # [P + Ts, nkv, hd]
    mean_v = v_all.mean(axis=0)                               # [nkv, hd]
    o = np.stack([mean_v[qh // (nq // nkv)] for qh in range(nq)]).reshape(-1)   # [nq * hd]
    want = h + gate_a * np.einsum("ok,k->o", lw["wo"], o)[None, :]
    got = oracle.dit_layer(h, lw, mod, kp, vp, pos, d)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)
    # the group map matters: a wrong head-to-group assignment changes the result
    o_bad = np.stack([mean_v[qh % nkv] for qh in range(nq)]).reshape(-1)
    bad = h + gate_a * np.einsum("ok,k->o", lw["wo"], o_bad)[None, :]
    assert np.max(np.abs(bad - got)) > 1e-6


# ----------------------------------------------------------------- INT8 weights (row-wise)

def test_int8_max_entry_maps_to_127_and_codes_are_bounded():
    w = RNG.standard_normal((64, 300)).astype(np.float32) * 0.02
    codes, scales = oracle.quantize_rowwise_int8(w)
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    assert codes.min() >= -127 and codes.max() <= 127
    amax = np.max(np.abs(w), axis=1)
    np.testing.assert_array_equal(scales, (amax / np.float32(127.0)).astype(np.float32))
    arg = np.argmax(np.abs(w), axis=1)
    np.testing.assert_array_equal(np.abs(codes[np.arange(64), arg]), 127)
    # the dequantisation error of every element is at most half a step
    err = np.abs(oracle.dequantize_rowwise_int8(codes, scales) - w.astype(np.float64))
    assert np.all(err <= scales.astype(np.float64)[:, None] * 0.5 * (1 + 1e-6))


def test_int8_integer_multiples_round_trip_and_ties_to_even():
    # scale 1 exactly (row max 127): integers round-trip, halves go to the even neighbour
    row = np.array([127.0, -127.0, 3.0, -64.0, 0.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 126.5], np.float32)
    codes, scales = oracle.quantize_rowwise_int8(row[None, :])
    assert scales[0] == np.float32(1.0)
    np.testing.assert_array_equal(codes[0], [127, -127, 3, -64, 0, 2, 4, -2, -4, 0, 0, 126])


def test_int8_zero_row_and_torch_round():
    w = RNG.standard_normal((8, 77)).astype(np.float32)
    w[3] = 0.0
    codes, scales = oracle.quantize_rowwise_int8(w)
    assert scales[3] == 1.0 and not codes[3].any()
    # torch.round is round-half-to-even on the same fp32 quotients
    q = torch.from_numpy(w) / torch.from_numpy(scales)[:, None]
    want = torch.clamp(torch.round(q), -127, 127).to(torch.int8).numpy()
    np.testing.assert_array_equal(codes, want)


# ----------------------------------------------------------------- INT4 weights (groups of 128)

def test_int4_groups_max_maps_to_7_and_ragged_last_group():
    w = RNG.standard_normal((16, 300)).astype(np.float32) * 0.02     # groups of 128, 128, 44
    codes, scales = oracle.quantize_groupwise_int4(w)
    assert codes.shape == (16, 300) and scales.shape == (16, 3)
    assert codes.min() >= -7 and codes.max() <= 7
    for g, (a, b) in enumerate(((0, 128), (128, 256), (256, 300))):
        amax = np.max(np.abs(w[:, a:b]), axis=1)
        np.testing.assert_array_equal(scales[:, g], (amax / np.float32(7.0)).astype(np.float32))
        arg = a + np.argmax(np.abs(w[:, a:b]), axis=1)
        np.testing.assert_array_equal(np.abs(codes[np.arange(16), arg]), 7)


def test_int4_ties_zero_group_and_torch():
    row = np.zeros((1, 256), np.float32)
    row[0, :8] = [7.0, -7.0, 2.5, 3.5, -2.5, 0.5, 1.5, 6.5]     # group 0: scale exactly 1
    codes, scales = oracle.quantize_groupwise_int4(row)
    assert scales[0, 0] == 1.0 and scales[0, 1] == 1.0             # group 1 is all zero
    np.testing.assert_array_equal(codes[0, :8], [7, -7, 2, 4, -2, 0, 2, 6])
    assert not codes[0, 128:].any()
    w = RNG.standard_normal((8, 256)).astype(np.float32)
    codes, scales = oracle.quantize_groupwise_int4(w)
    s = torch.from_numpy(scales).repeat_interleave(128, dim=1)
    want = torch.clamp(torch.round(torch.from_numpy(w) / s), -7, 7).to(torch.int8).numpy()
    np.testing.assert_array_equal(codes, want)
    # the dequantised weight is torch's bf16 cast of the fp32 product
    deq = oracle.dequantize_groupwise_int4(codes, scales)
    want_deq = (torch.from_numpy(codes).float() * s).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(deq, want_deq)
    assert np.all(np.abs(deq - w) <= s.numpy() * 0.5 * (1 + 2 ** -7) + 1e-30)


# ----------------------------------------------------------------- prefix K/V producer

def test_prefix_kv_invariants():
    rng = np.random.default_rng(21)
    P, Hv, nkv, hd = 9, 48, 2, 16
    h = rng.standard_normal((P, Hv))
    wk = rng.standard_normal((nkv * hd, Hv)) * 0.1
    wv = rng.standard_normal((nkv * hd, Hv)) * 0.1
    g = 1.0 + 0.1 * rng.standard_normal(Hv)
    k, v = oracle.prefix_kv(h, wk, wv, g, nkv)
    assert k.shape == (P, nkv, hd) and v.shape == (P, nkv, hd)
    # RMSNorm makes the result invariant to a per-token scale of h (eps = 0)
    k2, v2 = oracle.prefix_kv(h * np.linspace(0.5, 3.0, P)[:, None], wk, wv, g, nkv, eps=0.0)
    k0, v0 = oracle.prefix_kv(h, wk, wv, g, nkv, eps=0.0)
    np.testing.assert_allclose(k2, k0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v2, v0, rtol=1e-12, atol=1e-12)
    # position 0 is not rotated; every position keeps the per-pair norms of the projection
    x = h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + 1e-6) * g
    kp = (x @ wk.T).reshape(P, nkv, hd)
    np.testing.assert_allclose(k[0], kp[0], rtol=1e-12, atol=1e-12)
    pair = lambda a: a[..., : hd // 2] ** 2 + a[..., hd // 2:] ** 2
    np.testing.assert_allclose(pair(k), pair(kp), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v, (x @ wv.T).reshape(P, nkv, hd), rtol=1e-12, atol=1e-12)
