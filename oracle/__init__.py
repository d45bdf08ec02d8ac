"""CPU oracle for the flow-matching action-expert denoise loop.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library; the only module both sides use is ``synth`` (seeded inputs).

Everything is plain numpy in float64 on the bf16-rounded inputs.  A library
matmul serves as the dot-product step; there is no blocking, fusion or
reordering beyond the definitions below.

Functions and what pins them (tests under ``tests/test_oracle_*.py``):

=====================  =========================================================
``euler_integrate``    closed form of Euler on a linear field v = A x + b,
                       exact-ODE error bound, A = 0 and N = 1 special cases
``euler_integrate_grid`` the uniform grid reproduces ``euler_integrate``; a
                       skipped-step grid equals a brute-force velocity cache
                       (DP-Cache reading); first-order convergence on a graded
                       grid; the one-step grid; grid validation
``euler_integrate_switch`` closed form for two linear fields (matrix powers),
                       n_stale = 0 / N reduce to one field
``timestep_embedding`` t = 0 gives [1..1, 0..0]; first frequency is 1000 t;
                       last frequency matches the base-10000 geometric series
``adaln_table``        closed form at t = 0 (SiLU(1) x row sums of the cos half of
                       W_ada, plus b_ada)
``rms_norm``           unit RMS at eps = 0, scale invariance, torch's rms_norm
``modulate``           shift = scale = 0 is the identity
``rope_half``          per-pair norm, position 0 identity, relative-position
                       property, complex-multiplication form
``gqa_attention``      torch SDPA (enable_gqa) in float64, brute-force score
                       matrix, P = 0, constant-V rows, MHA case
``linear``/``swiglu``  torch float64 linear / silu, SiLU(0) = 0
``e4m3_*``             exhaustive code table, RNE ties, saturation, torch cast
``*_int4``             per 128-input group: the max entry maps to +-7, ties to
                       even, zero groups, ragged last group, torch's round on
                       the quotients and torch's bf16 cast of code * scale
``*_int8``             the max entry maps to +-127, integer multiples of the
                       scale round-trip, half-to-even ties, zero rows, torch's
                       round on the same quotients, |W' - W| <= scale / 2
``prefix_kv``          composed of the pinned rms_norm / linear / rope_half;
                       invariant to scaling h; position 0 is the plain projection
``dit_layer``          zero gates give the identity, joint prefix permutation
                       invariance, self-token permutation equivariance, branch
                       isolation under each adaLN gate, and the closed form of
                       uniform attention (W_q = 0: each head outputs the mean of
                       its kv group's prefix + self value rows)
``velocity``           closed form with every adaLN gate and the final
                       modulation zero (W_out RMSNorm(W_in x + b_in) + b_out on the
                       action rows, the state row dropped); one step of
                       ``denoise`` is one Euler update of it
``denoise``            batch independence (bitwise), determinism; the loop is
                       ``euler_integrate``'s, pinned above
=====================  =========================================================
"""

from .model import (  # noqa: F401
    bf16_to_f64, t_schedule, timestep_embedding, silu, rms_norm, modulate, rope_half,
    rope_positions_angles, gqa_attention, linear, swiglu, euler_integrate, euler_integrate_grid,
    check_t_grid, uniform_grid, euler_integrate_switch, denoise_stale, prefix_kv,
    adaln_table, dit_layer, embed_tokens, velocity, denoise, denoise_batch, OracleWeights,
)
from .fp8 import (  # noqa: F401
    e4m3_decode, e4m3_encode, quantize_rowwise_e4m3, dequantize_rowwise_e4m3,
)
from .int8 import quantize_rowwise_int8, dequantize_rowwise_int8  # noqa: F401
from .int4 import quantize_groupwise_int4, dequantize_groupwise_int4  # noqa: F401
