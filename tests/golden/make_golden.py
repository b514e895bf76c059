"""Writes tiny_oracle.json: a digest of the CPU oracle on the tiny workload.

Calls only the oracle (and the seeded input generator).  The digest guards the
oracle against unintended drift; the independent pins live in test_oracle.py.
Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from activation_sparse_gemm_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def digest():
    wl = WORKLOADS["tiny"]
    X, W, L_A, L_B = make_inputs(wl)
    meta, vals, s = oracle.sparsify(X)
    Y = oracle.linear(X, W, L_A, L_B)
    Yd = oracle.linear(X, W, mode=oracle.MODE_DENSE_SKIP)
    return {
        "workload": "tiny 128x256x256, R=64, seed 0",
        "inputs_sha256": hashlib.sha256(X.tobytes() + W.tobytes() + L_A.tobytes() + L_B.tobytes()).hexdigest(),
        "meta_sha256": hashlib.sha256(meta.tobytes()).hexdigest(),
        "vals_sha256": hashlib.sha256(vals.tobytes()).hexdigest(),
        "s_first16": [float(v) for v in s[:16]],
        "Y_diag16": [float(Y[i, i]) for i in range(16)],
        "Y_dense_diag16": [float(Yd[i, i]) for i in range(16)],
        "Y_fro": float(np.linalg.norm(Y)),
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(out, "w") as f:
        json.dump(digest(), f, indent=1)
    print("wrote", out)
