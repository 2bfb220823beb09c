"""Writes tests/golden/*.json by calling only the CPU oracle and the seeded
input generators.  The ELMO pages print no worked numeric example, so these
fixtures are regression records of the pinned oracle, not values from the
pages.  Re-run only when a change to the oracle's arithmetic is justified by
a reading of the pages; the commit must name that reading."""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from synthetic import make_labels, make_W_bf16, make_W_f32, make_X, workload  # noqa: E402


def sha(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def tiny_record(dtype):
    w = workload("tiny", dtype=dtype)
    X = make_X(w, 0)
    rowptr, cols = make_labels(w, 0)
    if dtype == "bf16":
        W = make_W_bf16(w)
    else:       # E4M3 codes; an E5M2 head starts from the same values rounded onto E5M2
        W = oracle.sr_round(make_W_f32(w), "e5m2" if dtype == "e5m2" else "fp8", seed=0, step=2**64 - 1)
    r = oracle.train_step(W, X, rowptr, cols, w.lr, 0, 0, dtype, want_zg=True, nthreads=1)
    return {
        "workload": "tiny (B=32, d=64, L=4096), lr=0.05, seed 0, step 0, dtype " + dtype,
        "W_in_sha256": sha(W), "W_out_sha256": sha(r["W"]),
        "G_sha256": sha(r["G"]),
        "dX_row0": [float(v) for v in r["dX"][0, :8]],
        "Z_label0": [float(v) for v in r["Z"][0, :8]],
    }


def kahan_record():
    """Three Kahan-compensated SGD steps of 4096 bf16 parameters."""
    rng = np.random.default_rng(7)
    bits = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)   # noqa: E731
    p, c = bits(rng.standard_normal(4096) * 0.05), np.zeros(4096, np.uint16)
    for _ in range(3):
        p, c = oracle.kahan_sgd(p, c, bits(rng.standard_normal(4096)), 1e-3)
    return {"p_sha256": sha(p), "c_sha256": sha(c), "p_first8": [int(v) for v in p[:8]]}


def main():
    x = (np.random.default_rng(8).standard_normal(4096) * 0.02).astype(np.float32)
    out = {"bf16": tiny_record("bf16"), "fp8": tiny_record("fp8"),
           "fp8_ge5m2": tiny_record("fp8_ge5m2"), "e5m2": tiny_record("e5m2"),
           "sr_draws_seed0_step0_first16": [int(k) for k in oracle.draw16(0, 0, 0, 16)],
           "sr_e5m2_seed3_step4_sha256": sha(oracle.sr_round(x, "e5m2", 3, 4)),
           "kahan": kahan_record()}
    with open(os.path.join(HERE, "tiny_step.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
