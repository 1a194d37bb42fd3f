"""Write tests/golden/tiny_oracle_digest.json from the CPU oracle alone.

The pages (the RFQ paper and its summaries) print no worked example, so this
fixture is not from them: it records what the pinned oracle produces for the
tiny RFQ linear workload (X 128x256 N(0,1) with channels 7 and 100 scaled x64,
W 128x256 N(0, 0.02), seed 0), so that any later change to the oracle's
arithmetic shows up as a diff here and has to be justified.

Run:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_scaled_gemm_rfq_b200 import workloads as wl  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def compute():
    w = wl.tiny(0)
    qa = oracle.quantize_bf16(w.x_bits, residual=True)
    qw = oracle.quantize_bf16(w.w_bits, residual=False)
    Y, S, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=True)
    Yoff, Soff, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=False)
    return {
        "workload": w.name,
        "seed": w.seed,
        "x_bits_sha256": digest(w.x_bits),
        "w_bits_sha256": digest(w.w_bits),
        "codes_x_sha256": digest(qa["codes_x"]),
        "scales_x_sha256": digest(qa["scales_x"]),
        "codes_r_sha256": digest(qa["codes_r"]),
        "scales_r_sha256": digest(qa["scales_r"]),
        "codes_w_sha256": digest(qw["codes_x"]),
        "scales_w_sha256": digest(qw["scales_x"]),
        "mma_scales_x_sha256": digest(oracle.scales_to_mma_layout(qa["scales_x"])),
        "S": S,
        "S_rfq_off": Soff,
        "Y_00": float(Y[0, 0]),
        "Y_127_127": float(Y[127, 127]),
        "Y_sum": float(Y.sum()),
        "Y_off_sum": float(Yoff.sum()),
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_digest.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1, sort_keys=True)
        f.write("\n")
    print("wrote", out)
