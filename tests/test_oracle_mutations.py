"""Plant one mistake at a time in the oracle (a compile-time switch in
oracle.c) and check that at least one pin fails for each.  This shows the
pins would catch a plausible bug in the oracle: a window or causal edge off by
one, a strided GQA head mapping, swapped cache axes, a dropped scale, a sign
error in the exponent, the wrong q8_0 group scale, or a dropped term in the
log-sum-exp, the wrong int8 row scale, a quantiser or fp16 conversion that
truncates, or new tokens written one slot off."""
import os
import tempfile

import pytest

import oracle
import pins

PLANTS = {
    1: "window one key too wide",
    2: "causal edge off by one",
    3: "query head -> KV head strided instead of grouped",
    4: "cache block and head axes swapped",
    5: "softmax scale dropped",
    6: "exponent sign flipped",
    7: "q8_0 scale of the wrong group",
    8: "max term dropped from lse",
    9: "int8 row scale of the neighbouring slot",
    10: "quantiser rounds toward zero",
    11: "cache write positions off by one",
    12: "fp32 -> fp16 truncates",
}

# The quick checks (skip the 65536-pattern fp16 decode, which no plant touches).
CHECKS = [c for c in pins.ALL_CHECKS if c is not pins.check_half_decode]


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=lambda p: PLANTS[p].replace(" ", "_"))
def test_planted_mistake_is_caught(plant):
    with tempfile.TemporaryDirectory() as d:
        path = oracle.build(plant=plant, out=os.path.join(d, f"liboracle_p{plant}.so"),
                            openmp=False)
        orc = oracle.load(path)
        caught = []
        for check in CHECKS:
            try:
                check(orc)
            except (AssertionError, oracle.OracleError):
                caught.append(check.__name__)
        assert caught, f"planted mistake '{PLANTS[plant]}' passed every pin"
