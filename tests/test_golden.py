"""The oracle reproduces its committed regression record (tests/golden)."""
import hashlib
import json
import os

import numpy as np
import pytest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_step_record(orc):
    from tests.golden.make_golden import kahan_record, sha, tiny_record
    ref = json.load(open(os.path.join(HERE, "tiny_step.json")))
    for dt in ("bf16", "fp8", "fp8_ge5m2", "e5m2"):
        assert tiny_record(dt) == ref[dt], dt
    assert [int(k) for k in orc.draw16(0, 0, 0, 16)] == ref["sr_draws_seed0_step0_first16"]
    x = (np.random.default_rng(8).standard_normal(4096) * 0.02).astype(np.float32)
    assert sha(orc.sr_round(x, "e5m2", 3, 4)) == ref["sr_e5m2_seed3_step4_sha256"]
    assert kahan_record() == ref["kahan"]
