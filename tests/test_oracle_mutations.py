"""Planted mistakes in a copy of the oracle must be caught by the independent pins.

Each mutation edits the oracle's source text (on the CPU, in memory) and loads
the edited copy as a separate module; the brute-force and closed-form checks
from the pin tests must then fail. This shows that a dropped term, a wrong sign
or index, or a transposed operand anywhere in the oracle would not go unnoticed.
"""
import importlib.util
import inspect
import types

import numpy as np
import pytest

from oracle import vda_oracle as vo
from tests import test_oracle_pins as pins

MUTATIONS = {
    "drop_alpha": ("return alpha[:, None] * P, B @ P", "return P, B @ P"),
    "alpha_on_right": ("return alpha[:, None] * P, B @ P", "return P * alpha[None, :], B @ P"),
    "transpose_B": ("return alpha[:, None] * P, B @ P", "return alpha[:, None] * P, B.T @ P"),
    "drop_identity": ("P = np.linalg.solve(np.eye(d_k) + A, np.eye(d_k))",
                      "P = np.linalg.solve(A + 1e-3 * np.eye(d_k), np.eye(d_k))"),
    "stats_no_beta": ("bK = Kf * beta[:, None]", "bK = Kf"),
    "stats_swap": ("return Kf.T @ bK, Vf.T @ bK", "return Kf.T @ bK, bK.T @ Vf"),
    "text_full_init": ("F = forward_scan(M, C, S_T / 2.0", "F = forward_scan(M, C, S_T"),
    "fwd_index": ("S_fwd.append(F[max(0, c * (j - 1) - 1)])", "S_fwd.append(F[max(0, c * (j - 1))])"),
    "rev_index": ("S_rev.append(R[min(T - 1, c * (j + 2))])", "S_rev.append(R[min(T - 1, c * (j + 2) - 1)])"),
    "readout_transposed": ("o = Qh[t] @ S.T", "o = Qh[t] @ S"),
    "scan_includes_anchor": ("range(1, T - 1))\n        R", "range(0, T - 1))\n        R"),
    "text_state_transposed": ("np.linalg.solve(np.eye(d_k) + A_txt, B_txt.T).T",
                              "np.linalg.solve(np.eye(d_k) + A_txt, B_txt.T)"),
    "chunk_offset": ("return t // c", "return (t + 1) // c"),
    "rms_mean_vs_sum": ("np.mean(o * o, axis=-1, keepdims=True)", "np.sum(o * o, axis=-1, keepdims=True)"),
    "gate_sign": ("return r * (1.0 / (1.0 + np.exp(-g)))", "return r * (1.0 / (1.0 + np.exp(g)))"),
    "conv_flip": ("out += xp[:, a:a + gh, b:b + gw, :] * w[:, a, b]",
                  "out += xp[:, a:a + gh, b:b + gw, :] * w[:, 4 - a, 4 - b]"),
    "temporal_causal": ("out += xp[s:s + T] * w[:, s]", "out += xp[s:s + T] * w[:, 4 - s]"),
    "silu_sign": ("return x / (1.0 + np.exp(-x))", "return x / (1.0 + np.exp(x))"),
}


def _mutant(name):
    src = inspect.getsource(vo)
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, name
    mod = types.ModuleType("vda_oracle_mutant_" + name)
    # The first occurrence is the forward path's (the frame-step backward, further
    # down, repeats some lines and has pins of its own).
    exec(compile(src.replace(old, new, 1), mod.__name__, "exec"), mod.__dict__)
    return mod


def _checks(mod):
    """Run the independent pins against ``mod``; return True if all pass."""
    ok = True
    saved = pins.vo
    pins.vo = mod
    try:
        for fn, args in [
            (pins.test_hand_derived_scalar_example, ()),
            (pins.test_whole_branch_matches_bruteforce, (0, 8, 2)),
            (pins.test_whole_branch_matches_bruteforce, (1, 9, 3)),
            (pins.test_text_counted_once, ()),
            (pins.test_frame_solve_matches_bruteforce_least_squares, (3,)),
            (pins.test_prep_branch_matches_bruteforce, ()),
            (pins.test_separable_conv_matches_torch_conv3d, ()),
            (pins.test_norms_closed_forms, ()),
        ]:
            try:
                fn(*args)
            except (AssertionError, KeyError, IndexError, ValueError, np.linalg.LinAlgError):
                ok = False
    finally:
        pins.vo = saved
    return ok


def test_unmutated_copy_passes():
    src = inspect.getsource(vo)
    mod = types.ModuleType("vda_oracle_copy")
    exec(compile(src, mod.__name__, "exec"), mod.__dict__)
    assert _checks(mod)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    assert not _checks(_mutant(name)), f"mutation {name} slipped through the pins"
