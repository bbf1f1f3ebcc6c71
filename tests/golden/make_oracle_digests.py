"""Write oracle_digests.json: SHA-256 digests of the oracle's outputs on a tiny
seeded case, one per step of the path (calls only oracle/ and the seeded input
generator).

The pages print no worked example, so nothing here pins the oracle to the method:
the pins are the closed forms, brute force and invariants of tests/test_oracle_*.
This file only makes a change to the oracle's arithmetic visible: a test compares
the digests, and a regenerated file belongs in a commit that names the passage, or
the reading of it, that justifies the change.

    python tests/golden/make_oracle_digests.py
"""
import hashlib
import json
import math
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from bit_fp8_attention_prep_b200 import synth  # noqa: E402

CASE = dict(B=1, S=300, H=1, k=4, iters=3, seed=0, rows=[0, 1, 127, 128, 255, 299])


def _digest(a):
    a = np.ascontiguousarray(a)
    return hashlib.sha256(a.dtype.str.encode() + str(a.shape).encode() + a.tobytes()).hexdigest()[:32]


def compute():
    c = CASE
    Q, K, V = synth.make_qkv(c["B"], c["S"], c["H"], recipe="mixture", seed=c["seed"])
    q, k, v = (X[0, :, 0].float().numpy() for X in (Q, K, V))
    out = {}
    prep = O.prepare_v_head(v, c["k"], c["iters"], c["seed"], 0)
    out["assign"] = _digest(np.asarray(prep["assign"], np.int64))
    out["perm"] = _digest(prep["perm"])
    out["mu"] = _digest(prep["mu"])
    out["v_codes_e4m3"] = _digest(prep["v_codes"])
    out["s_v"] = _digest(np.asarray([prep["s_v"]], np.float32))
    nv = O.prepare_v_head(v, c["k"], c["iters"], c["seed"], 0, fmt="nvfp4")
    out["v_codes_nvfp4"] = _digest(nv["v_codes"])
    out["v_scales_nvfp4"] = _digest(nv["v_scales"])
    qc, qs, kc, ks = O.quant_qk_head(q, k, prep["perm"])
    out["q_codes"], out["q_scales"] = _digest(qc), _digest(qs)
    out["k_codes"], out["k_scales"] = _digest(kc), _digest(ks)
    scale = 1.0 / math.sqrt(128)
    o, codes, M, l = O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], c["S"], c["rows"], scale,
                                         return_codes=True)
    out["p_codes"] = _digest(codes)
    out["frames"] = _digest(np.asarray(M))
    out["row_sums"] = _digest(np.asarray(l, np.float64))   # numpy's pairwise sum, no BLAS
    # O itself goes through a BLAS product whose summation order may follow the
    # thread count, so it is not digested
    out["residual_energy"] = _digest(np.asarray([O.residual_energy(v, prep["perm"], prep["mu"])], np.float64))
    return {"case": c, "digests": out}


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_digests.json"), "w") as f:
        json.dump(compute(), f, indent=1, sort_keys=True)
        f.write("\n")
    print("wrote", os.path.join(HERE, "oracle_digests.json"))
