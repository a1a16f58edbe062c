"""Each planted mistake in the oracle must be caught by at least one pin.

The oracle source carries ORACLE_MUTANT switches (off in the real build); this
test compiles each mutant into a temporary directory and runs the pin suite.
"""

import pytest

import oracle_pins
from oracle import Oracle

MUTANTS = {
    1: "block offset taken from the block index",
    2: "GQA heads interleaved (h % H_kv) instead of grouped (h / G)",
    3: "strict causal inequality",
    5: "softmax scale dropped",
    6: "softmax normalisation dropped",
    7: "speculative rows see the whole context",
    8: "values used in place of keys for the scores",
    9: "block-table rows packed by used length",
    10: "cache write one slot off",
    11: "bf16 widened with the wrong shift",
    12: "pool laid out head-major inside a block",
    13: "sliding window one key too long",
    41: "FP8 encode truncates instead of rounding to nearest",
    42: "FP8 exponent bias 8",
    43: "FP8 out-of-range values become NaN instead of saturating",
    31: "block copy leaves the value pool out",
    32: "block copy leaves the block's last token behind",
    33: "block copy with source and destination swapped",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_pins_catch_mutant(mutant, tmp_path_factory):
    out_dir = str(tmp_path_factory.mktemp(f"mutant{mutant}"))
    orc = Oracle(mutant=mutant, out_dir=out_dir)
    assert orc.lib.oracle_mutant_id() == mutant
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, ValueError) as exc:  # ValueError: oracle status != 0
            caught.append((check.__name__, str(exc)[:80]))
    assert caught, f"no pin caught mutant {mutant}: {MUTANTS[mutant]}"
