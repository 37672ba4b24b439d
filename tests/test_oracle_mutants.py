"""Planted mistakes in the NumPy twin must be caught by the pins.

Each mutant replaces one named step of ``oracle/np_oracle.py`` with a plausible error (a
wrong rounding rule, a dropped term, a wrong sign, an off-by-one denominator, a flipped
bit order); the listed pin must then fail.  This shows that the pins constrain every
step, not only the happy path.
"""
import numpy as np
import pytest

import oracle_pins as P
from oracle import np_oracle as no
from oracle_impls import NpOracle


def _rn_bf16(c):
    u = c.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


MUTANTS = {
    "round_half_up": ("_rne", lambda x: np.floor(x + np.float32(0.5)), [P.pin_quant_ties_half_even]),
    "scale_over_2^b": ("_scale_divisor", lambda b: (1 << b).astype(np.float32), [P.pin_quant_exact_grid]),
    "zero_not_clamped": ("_zero_point", lambda wmin, sf, L: np.rint(-wmin / sf),
                         [P.pin_quant_clamped_zero]),
    "symmetric_zero": ("_zero_point", lambda wmin, sf, L: np.floor((L + 1) / 2).astype(np.float32),
                       [P.pin_quant_zero_tie, P.pin_quant_bruteforce]),
    "cell_without_margin": ("_cell_halfwidth_f32", lambda sf: np.float32(0.5) * sf,
                            [P.pin_projected_residual_f32]),
    "bf16_bound_rounded_nearest": ("_bf16_bound", _rn_bf16, [P.pin_projected_residual_bf16]),
    "verify_drops_residual": ("_served_weight", lambda sf, k, r: sf * k, [P.pin_negative_control]),
    "dequant_zero_sign": ("_dequant_f64", lambda s, q, z: s * (q + z), [P.pin_matmul]),
    "msb_first": ("_BIT_ORDER", "big", [P.pin_pack_lsb_first]),
    "reparam_without_sqrt": ("_reparam_phi", lambda t: (np.asarray(t, np.float32) /
                                                       (np.float32(1) + np.asarray(t, np.float32) ** 2)),
                             [P.pin_reparam_closed_forms, P.pin_reparam_stays_in_cell]),
    "reparam_derivative_power": ("_reparam_dphi", lambda t: (np.float32(1) / np.sqrt(
                                     np.float32(1) + np.asarray(t, np.float32) ** 2)).astype(np.float32),
                                 [P.pin_reparam_gradient]),
    "reparam_nan_kept": ("_reparam_phi", lambda t: np.clip(np.asarray(t, np.float32) / np.sqrt(
                             np.float32(1) + np.asarray(t, np.float32) ** 2), -1, 1).astype(np.float32),
                         [P.pin_reparam_stays_in_cell]),
    "reparam_bf16_bound_rounded_nearest": ("_reparam_bound", lambda s, dt: _rn_bf16(no._halfwidth(s)) if dt == "bf16"
                                           else no._halfwidth(s), [P.pin_reparam_stays_in_cell]),
    "requant_accepts_ties": ("_rq_accept", lambda up, down, q, L: (1 if (q < L and up <= 0.0) else
                                                               (-1 if (q > 0 and down <= 0.0) else 0)),
                             [P.pin_requant_weight_space_is_rtn]),
    "requant_change_sign": ("_rq_changes", lambda sk, hkk, gk: ((sk * sk) * hkk + (2.0 * sk) * gk,
                                                                (sk * sk) * hkk - (2.0 * sk) * gk),
                            [P.pin_requant_strictly_lowers_output_error]),
    "requant_stale_gradient": ("_rq_update", lambda g, delta, hk: g, [P.pin_requant_local_optimum]),
    "index_rank_from_the_end": ("_width_rank", lambda sel: sel.sum() - np.cumsum(sel),
                                [P.pin_index_hand_example]),
    "rrq_residual_sign": ("_rrq_residual", lambda r, deq: r + deq,
                          [P.pin_rrq_residual_inside_half_step, P.pin_rrq_telescopes]),
    "rrq_residual_not_updated": ("_rrq_residual", lambda r, deq: r + np.float32(0) * deq,
                                 [P.pin_rrq_telescopes, P.pin_rrq_on_grid_is_exact]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, repl, pins = MUTANTS[name]
    monkeypatch.setattr(no, attr, repl)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin(NpOracle())
