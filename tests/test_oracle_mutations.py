"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/compressor.py`` (on the CPU,
never in the library), points the pin tests at the planted copy and checks that
at least one pin fails. A mistake no pin notices would mean the pins leave that
part of the oracle unchecked.
"""

import os
import sys
import types

import pytest

import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "compressor.py")

MUTATIONS = {
    "ape dropped": (
        "sc = sc + np.asarray(ape, dtype=np.float64)[np.asarray(positions, dtype=np.int64) % ratio]",
        "sc = sc + 0.0 * np.asarray(ape, dtype=np.float64)[np.asarray(positions, dtype=np.int64) % ratio]"),
    "ape row shifted": (
        "[np.asarray(positions, dtype=np.int64) % ratio]",
        "[(np.asarray(positions, dtype=np.int64) + 1) % ratio]"),
    "a/b halves swapped": (
        "K = np.where(use_b[None, :, None], K[..., D:], K[..., :D])",
        "K = np.where(use_b[None, :, None], K[..., :D], K[..., D:])"),
    "masked rows get score 0": (
        "Z = np.full(pos.shape + (C,), -np.inf, dtype=np.float64)",
        "Z = np.full(pos.shape + (C,), 0.0, dtype=np.float64)"),
    "previous window taken from the current one": (
        "pos = np.concatenate([(w - 1) * ratio + j, w * ratio + j], axis=1)",
        "pos = np.concatenate([w * ratio + j, w * ratio + j], axis=1)"),
    "softmax over channels": (
        "m = Z.max(axis=1, keepdims=True)\n    p = np.exp(Z - m)\n    return (p * K).sum(axis=1) / p.sum(axis=1)",
        "m = Z.max(axis=2, keepdims=True)\n    p = np.exp(Z - m)\n    return (p * K).sum(axis=1) / p.sum(axis=1)"),
    "softmax weights not normalised": (
        "return (p * K).sum(axis=1) / p.sum(axis=1)",
        "return (p * K).sum(axis=1)"),
    "rmsnorm eps dropped": (
        "np.mean(y * y, axis=-1, keepdims=True) + RMS_EPS", "np.mean(y * y, axis=-1, keepdims=True)"),
    "rmsnorm sum instead of mean": (
        "np.mean(y * y, axis=-1, keepdims=True)", "np.sum(y * y, axis=-1, keepdims=True)"),
    "rmsnorm weight dropped": ("+ RMS_EPS) * g", "+ RMS_EPS)"),
    "rope sign": ("ev * c[:, :h] - od * s[:, :h]", "ev * c[:, :h] + od * s[:, :h]"),
    "rope pairs halves instead of interleaved": (
        "    ev = z[:, D - rope_head_dim::2]\n    od = z[:, D - rope_head_dim + 1::2]",
        "    ev = z[:, D - rope_head_dim:D - h]\n    od = z[:, D - h:]"),
    "rope on the first channels": (
        "    out[:, D - rope_head_dim::2] = ev",
        "    out[:, 0:rope_head_dim:2] = ev"),
    "hadamard transposed": ("return z @ bf16_to_f64(hadamard_bits)",
                            "return z @ bf16_to_f64(hadamard_bits).T"),
    "tail threshold one window early": (
        "thr = (e // ratio - coff + 1) * ratio", "thr = (e // ratio - coff) * ratio"),
    "tail threshold one window late": (
        "thr = (e // ratio - coff + 1) * ratio", "thr = (e // ratio - coff + 2) * ratio"),
    "trigger one token late": ("nw = e // ratio - w0", "nw = (e - 1) // ratio - w0"),
    "row capacity too small": ("cap = np.minimum(L, L // ratio + 1)", "cap = np.minimum(L, L // ratio)"),
    "score history read through the kv table": (
        "r, o = self.slot(a[\"state_block_table\"], pos[hist])",
        "r, o = self.slot(a[\"kv_block_table\"], pos[hist])"),
    "slot offset by block instead of position": (
        "return rows, np.asarray(pos, dtype=np.int64) % bs",
        "return rows, (np.asarray(pos, dtype=np.int64) // bs) % bs"),
    "projection rounded to bf16 instead of fp32": (
        "return kv.astype(np.float32), sc.astype(np.float32)",
        "return f64_to_bf16_bits(kv).astype(np.uint32).__lshift__(16).view(np.float32), sc.astype(np.float32)"),
}

PIN_TESTS = [
    ("test_golden_ratio2_closed_form", {}),
    ("test_equal_scores_give_window_mean", {"ratio": 4}),
    ("test_equal_scores_give_window_mean", {"ratio": 128}),
    ("test_one_dominant_score_selects_its_row", {"ratio": 4}),
    ("test_first_c4a_window_ignores_previous_half", {}),
    ("test_rmsnorm_unit_rms_with_unit_weight", {}),
    ("test_rope_quarter_turn_and_identity", {}),
    ("test_hadamard_rotation_closed_forms", {}),
    ("test_layout_against_trigger_enumeration", {}),
    ("test_update_only_call_writes_state_and_zero_output", {}),
    ("test_ratio2_streaming_example", {}),
    ("test_tail_rule_is_exactly_what_later_calls_read", {"ratio": 4}),
    ("test_reordering_requests_does_not_change_results", {}),
] + [("test_oracle_matches_brute_force", {"case": c}) for c in pins.BRUTE_CASES]


def _load_mutant(old, new):
    src = open(SRC, encoding="utf-8").read()
    assert old in src, "mutation anchor not found"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    sys.modules["oracle_mutant"] = mod      # dataclasses look their module up by name
    try:
        exec(compile(src.replace(old, new, 1), SRC, "exec"), mod.__dict__)
    finally:
        sys.modules.pop("oracle_mutant", None)
    return mod


def _pins_fail(mod, monkeypatch):
    for name in ("compressor", "run_inputs", "layout", "out_rows", "window_row_positions",
                 "bf16_to_f64", "f64_to_bf16_bits"):
        monkeypatch.setattr(pins, name, getattr(mod, name))
    monkeypatch.setattr(pins.oracle, "compressor", mod)
    for test, kw in PIN_TESTS:
        try:
            getattr(pins, test)(**kw)
        except Exception:  # noqa: BLE001 - any failure (assertion or crash) catches the mutant
            return test
    return None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    mod = _load_mutant(*MUTATIONS[name])
    caught = _pins_fail(mod, monkeypatch)
    assert caught is not None, f"no pin notices: {name}"


def test_unmutated_copy_passes_all_pins(monkeypatch):
    mod = _load_mutant("RMS_EPS = 1e-6", "RMS_EPS = 1e-6")
    assert _pins_fail(mod, monkeypatch) is None
