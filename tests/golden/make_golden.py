"""Write the oracle regression fixtures in this folder.  Calls only the fp64 oracle (oracle/) on
seeded inputs from the shared generator; run from the repository root:
    python tests/golden/make_golden.py
The pages print no worked numeric example of the scan, so no fixture here comes from them; these
files only freeze the oracle's present output so that an unintended change to its arithmetic
shows up as a test failure (a deliberate change regenerates them and says why in its commit)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from selective_state_space_23_b200.inputs import make_inputs, to_f64, workload  # noqa: E402


def fixture():
    w = workload("tiny_f32", dim=4, seqlen=24, dstate=5)
    x = make_inputs(w, seed=99, with_dout=True, with_h0=True)
    f = {k: to_f64(v) for k, v in x.items()}
    fwd = oracle.scan_fwd(f["u"], f["delta"], f["A"], f["B"], f["C"], D=f["D"], z=f["z"],
                          dt_bias=f["dt_bias"], h0=f["h0"])
    bwd = oracle.scan_bwd(f["u"], f["delta"], f["A"], f["B"], f["C"], f["dout"], D=f["D"], z=f["z"],
                          dt_bias=f["dt_bias"], h0=f["h0"])
    return {
        "workload": {"batch": w.batch, "dim": w.dim, "seqlen": w.seqlen, "dstate": w.dstate,
                     "seed": 99, "io": "float32"},
        "out": fwd["out"].ravel().tolist(),
        "hL": fwd["hL"].ravel().tolist(),
        "grads": {k: v.ravel().tolist() for k, v in bwd.items() if v is not None},
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_tiny_seed99.json"), "w") as fh:
        json.dump(fixture(), fh)
    print("wrote oracle_tiny_seed99.json")
