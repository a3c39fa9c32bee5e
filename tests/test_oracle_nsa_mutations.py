"""The NsaCompressWithCache oracle's pins catch plausible mistakes: each case
plants one mistake in a copy of ``oracle/nsa.py`` (on the CPU), points the pin
tests at it and checks that at least one pin fails. The brute-force
restatement the pins compare with stays the original."""

import os
import sys
import types

import pytest

import tests.test_oracle_nsa as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "nsa.py")

MUTATIONS = {
    "window one token early": ("p = idx * stride + j\n", "p = idx * stride + j - 1\n"),
    "heads of the weight reversed": ("prod = to_f64(tok, dtype) * w[j][:, None]",
                                     "prod = to_f64(tok, dtype) * w[j][::-1][:, None]"),
    "trigger ignores the stride": (
        "return s >= compress_block_size and (s - compress_block_size) % stride == 0",
        "return s >= compress_block_size"),
    "packed rows of the next batch": ("tok = inp[int(start[b]) + p]", "tok = inp[int(start[min(b + 1, B)]) + p]"),
    "page offset by block": ("tok = inp[blk, p % page_block_size]",
                             "tok = inp[blk, (p // page_block_size) % page_block_size]"),
    "fp16 rounded like bf16": (
        "return f64_to_half_bits(v) if dtype == \"fp16\" else f64_to_bf16_bits(v)",
        "return f64_to_half_bits(np.asarray(v) * (1 + 2 ** -9)) if dtype == \"fp16\" else f64_to_bf16_bits(v)"),
    "slot of the next batch": ("slot = int(slots[b])", "slot = int(slots[(b + 1) % B])"),
}

PIN_TESTS = ["test_pages_example", "test_trigger_rule_and_untouched_slots",
             "test_paged_and_packed_layouts_agree"] + [
    ("test_one_hot_weight_copies_a_token", {"dtype": d}) for d in ("fp16", "bf16")] + [
    ("test_power_of_two_weight_scales_exactly", {"dtype": d}) for d in ("fp16", "bf16")] + [
    ("test_brute_force_tiny", {"dtype": d, "layout": l, "cbs": c, "stride": s, "pbs": p})
    for d in ("fp16", "bf16") for l in ("paged", "TND") for c, s, p in ((32, 16, 64), (48, 32, 64))]


def _load_mutant(old, new):
    src = open(SRC, encoding="utf-8").read()
    assert old in src, "mutation anchor not found"
    src = src.replace(old, new, 1).replace("from .compressor import", "from oracle.compressor import")
    mod = types.ModuleType("oracle_nsa_mutant")
    mod.__file__ = SRC
    sys.modules["oracle_nsa_mutant"] = mod   # dataclasses look their module up by name
    try:
        exec(compile(src, SRC, "exec"), mod.__dict__)
    finally:
        sys.modules.pop("oracle_nsa_mutant", None)
    return mod


def _pins_fail(mod, monkeypatch):
    for name in ("nsa_compress", "half_to_f64", "to_f64", "triggers"):
        monkeypatch.setattr(pins, name, getattr(mod, name))
    for t in PIN_TESTS:
        test, kw = (t, {}) if isinstance(t, str) else t
        try:
            getattr(pins, test)(**kw)
        except Exception:  # noqa: BLE001 - any failure (assertion or crash) catches the mutant
            return test
    return None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    caught = _pins_fail(_load_mutant(*MUTATIONS[name]), monkeypatch)
    assert caught is not None, f"no pin notices: {name}"


def test_unmutated_copy_passes_all_pins(monkeypatch):
    assert _pins_fail(_load_mutant("import dataclasses", "import dataclasses"), monkeypatch) is None
