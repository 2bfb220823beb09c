"""The oracle reproduces its committed regression record (tests/golden)."""
import hashlib
import json
import os

import numpy as np
import pytest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_step_record(orc):
    from tests.golden.make_golden import tiny_record
    ref = json.load(open(os.path.join(HERE, "tiny_step.json")))
    for dt in ("bf16", "fp8"):
        assert tiny_record(dt) == ref[dt]
    assert [int(k) for k in orc.draw16(0, 0, 0, 16)] == ref["sr_draws_seed0_step0_first16"]
