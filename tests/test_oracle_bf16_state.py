"""Pins of the reduced-precision (bfloat16) decode-state oracle: the rounding function against
torch's float32 -> bfloat16 conversion (round to nearest even) and hand-checked ties, and the step
against the float32-state step it rounds."""

import numpy as np
import torch

import oracle
import wkv7_inputs as wi


def test_round_bf16_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(100000, generator=g) * 10 ** e for e in range(-6, 7)])
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(x.to(torch.float64).numpy())
    assert np.array_equal(got, ref)


def test_round_bf16_ties_go_to_even():
    ulp = 2.0 ** -7  # spacing of bfloat16 in [1, 2)
    cases = {1.0 + ulp / 2: 1.0, 1.0 + 3 * ulp / 2: 1.0 + 2 * ulp, -(1.0 + ulp / 2): -1.0,
             1.0 + ulp / 2 + 2.0 ** -30: 1.0 + ulp, 0.0: 0.0, 2.0 - ulp / 2: 2.0}
    for x, want in cases.items():
        assert oracle.round_bf16(np.array([x]))[0] == want, x


def test_step_is_the_float64_step_rounded():
    d = wi.draw(3, 1, 4, seed=5, s0_std=0.1)
    s0 = oracle.round_bf16(d["s0"].numpy())
    ops = [d[n + "_f32"][:, 0] for n in ("r", "w", "k", "v", "a", "b")]
    y, s1 = oracle.decode_step_bf16_state(*ops, s0)
    y_ref, s_ref = oracle.wkv7(*[d[n + "_f32"] for n in ("r", "w", "k", "v", "a", "b")], s0, precision="f64")
    assert np.array_equal(y, y_ref[:, 0])
    assert np.array_equal(s1, oracle.round_bf16(s_ref))
    # every new state value is a bfloat16 value within half an ulp of the float64 state
    assert np.array_equal(oracle.round_bf16(s1), s1)
    assert np.all(np.abs(s1 - s_ref) <= 2.0 ** -8 * np.abs(s_ref))
