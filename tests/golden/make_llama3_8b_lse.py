"""Write linear_ce_llama3_8b_lse.npz: the oracle's lse of every row of the
Llama-3-8B head workload (inputs bf16 [16384, 4096], weight bf16 [128256,
4096], seed 0), which the full-size parity test needs and which takes about
17 TFLOP of float64 work to recompute.

Calls only the seeded input generator (gh_synth) and the oracle
(oracle.row_lse).  The file also records a SHA-256 digest of the input bytes,
so the test can confirm it was made from the inputs it regenerates.

    python tests/golden/make_llama3_8b_lse.py
"""
import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import gh_synth  # noqa: E402
import oracle  # noqa: E402

OUT = os.path.join(HERE, "linear_ce_llama3_8b_lse.npz")


def inputs_digest(p) -> str:
    h = hashlib.sha256()
    for a in (p.inputs, p.weight, p.targets):
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def main():
    t0 = time.time()
    p = gh_synth.linear_ce_llama3_8b()
    X = gh_synth.bf16_to_f32(p.inputs).astype(np.float64)
    W = gh_synth.bf16_to_f32(p.weight).astype(np.float64)
    lse = oracle.row_lse(X, W, row_block=512)
    np.savez_compressed(OUT, lse=lse, inputs_sha256=np.array(inputs_digest(p)), workload=np.array(p.name))
    print(f"wrote {OUT} ({time.time() - t0:.0f} s)")


if __name__ == "__main__":
    main()
