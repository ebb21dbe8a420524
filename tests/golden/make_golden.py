"""Write tests/golden/tiny_oracle.json from the oracle alone.

Run from the repository root: ``python tests/golden/make_golden.py``. It hashes the
seeded inputs of the 128-token workload and stores the oracle's fp64 outputs on
them, so that a drift of either the generator or the oracle shows up as a test
failure. Nothing here touches the CUDA library.
"""

import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from synthetic import make_inputs  # noqa: E402


def input_hashes(x):
    return {k: hashlib.sha256(np.ascontiguousarray(getattr(x, k)).tobytes()).hexdigest()
            for k in ("h_s", "h_t", "W_s", "W_t", "labels")}


def main():
    x = make_inputs("tiny", seed=0)
    f = oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau, side=True)
    b = oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, x.labels, x.beta, x.tau)
    out = {
        "source": "tests/golden/make_golden.py (oracle only), workload 'tiny', seed 0",
        "hashes": input_hashes(x),
        "loss_mean": f["loss_mean"],
        "n_valid": f["n_valid"],
        "loss_tok_first8_valid": [float(v) for v in f["loss_tok"][32:40]],
        "lse_s_first8_valid": [float(v) for v in f["lse_s"][32:40]],
        "lse_t_first8_valid": [float(v) for v in f["lse_t"][32:40]],
        "entropy_s_first8_valid": [float(v) for v in f["entropy_s"][32:40]],
        "logp_label_first8_valid": [float(v) for v in f["logp_label"][32:40]],
        "dh_s_fro": float(np.linalg.norm(b["dh_s"])),
        "dW_s_fro": float(np.linalg.norm(b["dW_s"])),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
